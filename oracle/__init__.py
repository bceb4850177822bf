"""CPU oracle for the reverse-KL loss: test infrastructure only.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference arm may import this package.  The product library never
does.  See ``rkl_oracle`` for the definitions and their sources.
"""
