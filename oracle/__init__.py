"""Plain CPU oracle for the NF4 QLoRA linear layer.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or
executes this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. It shares
no code, table or constant generator with the CUDA library; the two sides are
compared only through their outputs on the same seeded inputs.

Everything is written from the definitions, in numpy float64, with no blocking
or fusion beyond what the definitions state:

* ``nf4``    -- the NF4 codebook, blockwise absmax quantisation, nibble
                packing, double quantisation of the block constants and
                dequantisation to bf16 ("QLoRA, in depth", section "The
                mechanism in brief"; multigrid.ai "QLoRA", section "NF4 and
                double quantisation").
* ``linear`` -- the QLoRA linear forward y = W x + (alpha/r) B A x and its
                backward (dX, dA, dB, never dW) ("QLoRA, in depth", section
                "The mechanism in brief").
* ``sizes``  -- the storage ledger (bits per weight, packed bytes, LoRA
                parameter counts) that the pages quote.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against values the pages print, closed forms, brute force in exact rational
arithmetic, or library routines, except the choice of the NF4 offset constant,
which the pages do not fix (see ``nf4.NF4_OFFSET``: parity unpinned for that
one constant; the construction around it is pinned).
"""

from . import nf4, linear, sizes  # noqa: F401
