"""CPU oracle for the sparse-MoE FFN layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference leg of
``bench.py`` may import this package.  The product path (the CUDA library and its Python
binding) never imports, links or runs anything here, and shares no code with it.

Two independent restatements of the same definition live here:

* ``moe_oracle.c`` (plain C, double accumulation; loaded through ctypes) -- the oracle;
* ``moe_numpy.py`` (vectorised NumPy) -- a second restatement used to cross-check it.

Both follow the pages: "Step 3.5 Flash: Open Frontier-Level Intelligence with 11B Active
Parameters" sections 2.2 / 2.2.2 / 3.2.4 / 4.1.2, and the parameter table of "Step 3.5 Flash
技术论文深度解读" (architecture item 1).  See the header of ``moe_oracle.c``.
"""
from .c_oracle import (  # noqa: F401
    build_oracle,
    oracle_router_logits,
    oracle_route,
    oracle_gates,
    oracle_permute,
    oracle_expert_ffn,
    oracle_moe_forward,
    oracle_num_threads,
    oracle_set_num_threads,
    oracle_router_stats,
    oracle_bias_update,
    oracle_expert_act_rms,
    oracle_expert_param_norms,
    oracle_health_ratios,
    oracle_moe_backward,
    oracle_moe_backward_sampled,
)
