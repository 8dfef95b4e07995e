"""CPU oracle for absorbed MLA decode -- TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, float64 definition that the CUDA path is
checked against.  Only the test suite, the smoke check in
``__graft_entry__.py`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it.  The product path (the C-ABI library and its
Python binding) never imports, calls or links anything from here, and this
package never imports the product path: the two share no code.

Modules
-------
``mla_oracle``  un-absorbed (order 1) MLA decode attention in float64 NumPy,
                the order-2 (absorbed) intermediates, order 3 on tiny shapes,
                and a FLOP counter that instruments every contraction.
``brute``       pure-Python scalar loops of the same definition, for tiny
                shapes only (the brute-force pin of ``mla_oracle``).

Parity status of each function is stated in its docstring; nothing here is
"parity unpinned" except where a docstring says so.
"""
