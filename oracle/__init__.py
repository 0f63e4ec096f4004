"""Plain fp64 CPU oracle of head-scale KV-cache pruning for next-scale (VAR)
transformers (HeatKV).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
link this package: only the tests, the smoke check of the entry module and the
CPU-baseline leg of the benchmark use it.  It shares no code with the CUDA
library; the only module both sides use is the seeded input generator
(`synth`), which holds none of the method's arithmetic.

Every function is the plain definition of its step, written for a reader to
check against the sources by eye: NumPy fp64 arithmetic, a library matmul as
the only "primitive", Python loops for the index work.  No blocking, fusion or
reordering beyond what the definitions state.

Sources (cited by page title and section):
  [HeatKV]  "HeatKV: Head-tuned KV-cache Compression for Visual Autoregressive
            Modeling" project page -- Abstract, Method steps 1-5, Table 1.
  [Review]  the machine review page of the HeatKV paper (arXiv 2605.14877) --
            Figure 3 caption (raster order of a scale's tokens), Figure 4
            caption (Algorithm 1, BINARY-HEATKV / GREEDYEARLYPRUNING),
            Appendix A (Algorithm 2 header).
  [AMS-KV]  "AMS-KV: Adaptive KV Caching in Multi-Scale Visual Autoregressive
            Transformers" listing -- Abstract (local and condensed scales).

Parity status of each function is stated in its docstring; functions whose
result the pages do not fix exactly (the S-CAS formula) are pinned to the
library's stated definition and marked "parity unpinned" against the paper's
own S-CAS values, which the pages never print.
"""
from .scales import ScaleGeometry
from .attention import (block_causal_attention, attend, scas_mass, pruned_attention, attention_rows,
                        pruned_attention_rows)
from .schedule import scas_from_mass, build_schedule, BudgetError, full_cache_tokens
from .layout import build_offsets, compact_kv
from .generation import append_scale, cache_size_after_layer
from .stability import rank_stability, average_ranks
from .early_pruning import early_pruning_schedule, keep_after_step
from .quant import (quantize_block, dequantize_block, quantize_kv, quantize_block_int4, dequantize_block_int4,
                    pack_int4, unpack_int4, quantize_kv_int4, int4_scale_bits, quantize_block_int3,
                    dequantize_block_int3, pack_int3, unpack_int3, quantize_kv_int3, int3_scale_bits)

__all__ = [
    "ScaleGeometry", "block_causal_attention", "attend", "scas_mass", "pruned_attention",
    "attention_rows", "pruned_attention_rows", "scas_from_mass", "build_schedule", "BudgetError", "full_cache_tokens",
    "build_offsets", "compact_kv", "append_scale", "cache_size_after_layer",
    "rank_stability", "average_ranks", "early_pruning_schedule", "keep_after_step",
    "quantize_block", "dequantize_block", "quantize_kv", "quantize_block_int4", "dequantize_block_int4",
    "pack_int4", "unpack_int4", "quantize_kv_int4", "int4_scale_bits", "quantize_block_int3",
    "dequantize_block_int3", "pack_int3", "unpack_int3", "quantize_kv_int3", "int3_scale_bits",
]
