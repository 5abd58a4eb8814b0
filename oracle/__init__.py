"""CPU oracle for one decode step of the MFA (Multi-Matrix Factorization Attention) layer.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` use it.

The oracle is the plain definition of the layer, evaluated in float64 with numpy, written
from the Step-3 pages ("Step-3 is Large yet Affordable", bud-325 summary, sections
"Key claims" and "Method"; redeep.blog post, section "What's New" and the architecture
table). It shares no code, tables or constants with the CUDA path; the two meet only in
the seeded input generator ``decode_attention_10_b200.workloads``, which holds none of the
method's arithmetic.

Modules
-------
codecs  bf16 and OCP FP8 E4M3 encode/decode written from the two format definitions.
mfa     the layer: query down-projection, RMSNorm, query up-projection, K/V projection and
        cache append, 64-head attention over the shared K/V head, and their composition.

Parity status of each function is stated in its docstring ("pinned by ..."). The one part
with no pin is the whole layer against Step-3's real activations: the pages print none and
no weights are available ("parity unpinned" for that comparison only).
"""

from . import codecs, mfa  # noqa: F401
