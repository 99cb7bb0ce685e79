"""fp64 CPU oracle for the DHSA prefill path (test infrastructure only).

Imported by the test suite, the smoke check and the CPU-baseline leg of the
benchmark; never by the product path.
"""
