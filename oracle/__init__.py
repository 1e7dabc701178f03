"""CPU oracle for the grouped linear layer (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg use this
package; the library never imports it.
"""
