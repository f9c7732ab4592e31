"""CPU oracle for tile-routed FP16/INT8 attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call,
link or execute this package: only the tests, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm use it.  It shares no code with
the CUDA library; the two meet only through the seeded input generators.

Everything here is plain fp64 NumPy (plus exact integer arithmetic and the
fp32 steps that the quantiser definition fixes), written to be checked by eye
against the method it restates:

* TileMix (Lattice paper page "TileMix ..."), abstract: the attention matrix
  is cut into hardware-aligned score tiles, each group of ``g`` adjacent key
  tiles gets one routing bit packed in a compact bitmask, the group's scores
  are computed in FP16 or INT8, both paths feed one online-softmax state, all
  legal groups are computed (dense connectivity), and grouped-query attention,
  variable-length batches and INT8 key/value caches are supported.
* MLX PR "Nax Refactor" (ml-explore/mlx #3271), attention timing tables:
  fused scaled-dot-product attention in float16 with GQA and causal masking,
  and the FLOP convention of its ``tflops`` column.

Parity status of each function is stated in its docstring.  The only part
with "parity unpinned" is the model-quality frontier, which is not built.
"""

from .tilemix_oracle import (  # noqa: F401
    SPLITMIX_GAMMA,
    attention,
    attention_rows,
    build_mask,
    build_mask_scale_policy,
    E4M3_MAX,
    dequant_cache,
    e4m3_decode,
    e4m3_encode,
    last_visible_key,
    mask_bit,
    mask_words,
    n_groups,
    n_tiles,
    quantize_tiles,
    quantize_tiles_fp8,
    route_stats,
    seq_table,
    splitmix64,
    tile_table,
    visible,
)
