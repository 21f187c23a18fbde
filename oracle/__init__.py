"""Plain, slow CPU oracle for the QLoRA NF4 quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.
It shares no code, table or constant generator with the CUDA library; each
side derives the NF4 codebook on its own and the tests compare them.

Sources (the pages the method is taken from):
  * "QLoRA" milestone page (nlp-lineage), section "The idea": NF4 spacing
    (16 values, equal share of N(0,1), exact zero), blocks of 64 with a
    32-bit scale, double quantisation of the scales to 8 bits, and the layer
    equation Y = X·doubleDequant(c1, c2, W_NF4) + X·L1·L2 with only L1 and L2
    receiving weight gradients.
  * inferensys glossary "QLoRA", NF4 and double-quantisation paragraphs
    (scales become 8-bit floats) and the kernel paragraph (dequantise to
    BFloat16 for the matrix multiply).
  * tecyfy "What is QLoRA", section "The 3 tricks"; examadda "QLoRA",
    sections "The Core Idea" and "The Three Innovations".
  * examadda "QLoRA", "Practical Notes" (merging an adapter into a 4-bit
    base is lossy: dequantise first) and the paged-optimizer passages
    (``adapters.py``).
"""

from .nf4_oracle import *  # noqa: F401,F403
from .adapters import *  # noqa: F401,F403
