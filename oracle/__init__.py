"""Oracle for the vision-to-language projector: TEST INFRASTRUCTURE ONLY.

A plain, slow CPU restatement of what the projector path computes, in fp64,
written from the pages' own statement of the method and used to check the
CUDA path. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import, call or link anything in this package. It shares no
code with the CUDA library and imports nothing from it.

Contents
--------
``projector``  numpy fp64 definition of every step (unshuffle, LayerNorm, MLP,
               tile assembly, scatter) and the closed-form counts.
``brute.c``    scalar C restatement of the same steps by direct index formulas,
               used to cross-check ``projector`` on tiny grids.

Every function is pinned by a ``-m "not gpu"`` test against values the pages
print, closed forms, library special cases or brute force (see the module
docstrings). Nothing here is unpinned.
"""
