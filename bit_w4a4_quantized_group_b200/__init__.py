"""B200-native SVDQuant W4A4 + low-rank linear layer.

The compute path is the C-ABI library ``libsvdq.so`` (CUDA, sm_100a) built
from ``csrc/``; :mod:`.binding` marshals arguments to it.  Submodules are
imported lazily so that the seeded input generators (:mod:`.inputs`) can be
used without loading the CUDA library.
"""
