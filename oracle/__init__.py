"""CPU oracle of the SVDQuant W4A4 linear layer -- test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline /
reference leg may import this package.  The product path never does.
"""
