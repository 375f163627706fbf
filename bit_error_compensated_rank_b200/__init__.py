"""Echo's error-compensated 4-bit all-reduce on one B200.

The compute path is ``libecho.so`` (CUDA, sm_100a) behind a C ABI declared in
``include/echo.h``; :mod:`bit_error_compensated_rank_b200.echo` is its thin
ctypes binding and :mod:`bit_error_compensated_rank_b200.workloads` draws the
seeded synthetic inputs. Importing this package loads nothing; importing the
binding loads the CUDA library and fails loudly if it is missing.
"""
