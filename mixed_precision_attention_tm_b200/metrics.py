"""FLOP conventions used to report attention throughput.

MLX PR "Nax Refactor" (ml-explore/mlx #3271), attention timing tables: the
printed tflops column equals 4 * B * n_qh * qsl * ksl * hdim (halved when
causal) divided by the time of one call, the printed t_fus being the total of
64 calls.  This library reports the same 4*d FLOP per query-key pair but
counts only visible pairs (bottom-right causal), which equals the MLX count
for square causal shapes up to the diagonal.
"""


def mlx_flops(B, n_qh, qsl, ksl, hdim, causal):
    """FLOP of one fused attention call in the MLX table's convention."""
    f = 4.0 * B * n_qh * qsl * ksl * hdim
    return f / 2 if causal else f


def visible_pairs(Lq, Lk, causal):
    """Query-key pairs with j < Lk and (not causal or j <= i + Lk - Lq)."""
    if not causal:
        return Lq * Lk
    total = 0
    off = Lk - Lq
    # rows i with i + off >= Lk - 1 see all Lk keys; earlier rows see i + off + 1
    full_from = max(0, Lk - 1 - off)
    first = max(0, -off)                      # first row with a visible key
    if full_from > first:
        a, b = first + off + 1, (full_from - 1) + off + 1
        total += (a + b) * (full_from - first) // 2
    total += max(0, Lq - max(full_from, first)) * Lk
    return total


def algorithmic_flops(d, n_visible_pairs):
    """4*d FLOP per visible pair: 2d for QK^T (FP16 or INT8) and 2d for P.V."""
    return 4.0 * d * n_visible_pairs
