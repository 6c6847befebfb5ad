"""CPU oracle for the MiniMax-H3 block forward (test infrastructure only).

Imported by the tests, the package smoke check and the benchmark's CPU
baseline, never by the CUDA path.
"""
