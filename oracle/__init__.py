"""CPU oracle for the W4A8 GEMM path: test infrastructure, not product code."""
