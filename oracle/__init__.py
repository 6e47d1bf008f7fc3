"""fp64 CPU oracle of dynamic block-sparse prefill attention.

Test infrastructure only: the tests, the package smoke check and the
benchmark's CPU-baseline leg use it; the product path never imports it.
"""
