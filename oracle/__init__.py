"""fp64 CPU oracle for the HHR decode path.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
CPU-baseline leg of bench.py, never by the library.  It shares no code with
the CUDA path.
"""
