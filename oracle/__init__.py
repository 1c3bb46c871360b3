"""Float64 CPU oracle for BasisKV decode attention -- test infrastructure only.

Only the tests, the smoke check and the benchmark's CPU-baseline leg use this
package; the CUDA library never does.
"""
