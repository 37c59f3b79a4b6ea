"""CPU oracle of the CSA indexer step: TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import anything here.  The product package never does.
"""
