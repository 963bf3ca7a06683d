"""fp64 CPU oracle for the MoE layer with zero-computation experts.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The CUDA library never calls it, and it shares no code with the library.

Every function cites the passage it follows.  Citations name the LongCat-Flash
write-up "Meituan's large model goes viral for its speed" (itouyu.top, in
Japanese; the same text appears translated on kqgmpj.cn and dhxrcw.cn) and a
section of it.  That article prints the MoE formula's symbol glossary but the
formula itself is lost; the readings taken where it is silent are listed in
``moe_zc_ref``'s module docstring.
"""
from .moe_zc_ref import (  # noqa: F401
    router_logits,
    softmax,
    select_topk,
    route,
    swiglu_expert,
    forward,
    forward_rows,
    expert_load,
    zero_pick_fraction,
    Routing,
)
