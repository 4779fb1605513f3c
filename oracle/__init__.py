"""fp64 CPU oracle for the two-level sparse decode step -- test infrastructure only.

Only tests, the smoke check and the benchmark's CPU-baseline leg import this
package; the CUDA product path never does.
"""
