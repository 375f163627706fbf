"""CPU oracle for Echo's error-compensated 4-bit all-reduce (test
infrastructure: only the tests, the smoke check and the benchmark's CPU
baseline import it)."""
