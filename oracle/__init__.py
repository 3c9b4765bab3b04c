"""CPU oracle (test infrastructure only): fp64 restatement of SparSTAR block-sparse attention."""
