"""CPU oracle of the MoE-layer forward: test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import it. The CUDA library never does, and the oracle
imports nothing from the library.
"""
from .moe_oracle import (as_f64, capacity, combine, dense_reference, expert_ffn,  # noqa: F401
                         expert_of_slot, forward, forward_rows, gather_rows, grouped_ffn,
                         permute, route, router_logits, swiglu, topk_ids, topk_weights)
