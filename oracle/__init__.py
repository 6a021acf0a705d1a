"""CPU oracle for the 2:4 sparse path (test infrastructure only).

Imported by the tests, the package smoke check and the benchmark's CPU
baseline leg; never by the library path.
"""
