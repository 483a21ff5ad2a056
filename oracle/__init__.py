"""VBQ oracle package: test infrastructure only (tests, smoke check, CPU-baseline leg of the benchmark)."""
