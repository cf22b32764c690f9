"""Work counts of the KDA operator used by the benchmark's roofline figures.

FLOPs follow the per-head training-FLOP model of "Kimi Linear: An Expressive, Efficient Attention
Architecture" (paper-graph-ui walkthrough, §3.4 "FLOPs Accounting and Inference Strategy"):

    FLOPs_KDA(T; C, d) = 6 T d^2 + 3 T C d + T C^2          (per head)

with the page's worked example T = 4096, C = 64, d = 128 (about 517M; the exact value is
520,093,696). Two more counts are reported beside it: the count that excludes the masked
triangular halves of the C x C products, and the count of the tiles the tensor cores issue.

Bytes are the ALGORITHMIC minimum each call must move through HBM: every input element read once,
every output element written once, states read and written once.
"""
from __future__ import annotations


def eq13_flops(T: int, C: int, d: int) -> int:
    """Per-head FLOPs of the chunkwise algorithm (the walkthrough's Eq. 13)."""
    return 6 * T * d * d + 3 * T * C * d + T * C * C


def triangular_flops(T: int, C: int, d: int) -> float:
    """Per-head FLOPs with the masked halves of the C x C products left out:
    W.S, Q.S, K^T.V' (6 T d^2) + half of K K^T and Q K^T and of W/U = M.(G.K, V) and A_qk.V'
    (5 T C d) + the triangular inverse (~ T C^2 / 3)."""
    return 6 * T * d * d + 5 * T * C * d + T * C * C / 3.0


def issued_tile_flops(T: int, C: int, d: int) -> int:
    """Per-head FLOPs of full (unmasked) C x C tiles: 6 T d^2 + 10 T C d."""
    return 6 * T * d * d + 10 * T * C * d


def prefill_min_bytes(token_heads: int, num_seqs: int, H: int, Dk: int, Dv: int,
                      qkv_bytes: int, with_initial_state: bool, with_final_state: bool) -> int:
    """Minimum HBM bytes of one chunkwise prefill call: q, k, v, log_alpha (fp32), beta (fp32)
    read once; o written once; the fp32 states read / written once."""
    per_th = (2 * Dk + Dv) * qkv_bytes + 4 * Dk + 4 + Dv * qkv_bytes
    states = num_seqs * H * Dk * Dv * 4
    return token_heads * per_th + states * (int(with_initial_state) + int(with_final_state))


def decode_state_bytes(N: int, H: int, Dk: int, Dv: int) -> int:
    """fp32 state bytes one decode step must read and write (the metric's 'state GB/s')."""
    return 2 * N * H * Dk * Dv * 4


def decode_total_bytes(N: int, H: int, Dk: int, Dv: int, qkv_bytes: int) -> int:
    """All bytes of one decode step: state in/out, q, k, v, log_alpha, beta in, o out."""
    per_head = (2 * Dk + Dv) * qkv_bytes + 4 * Dk + 4 + Dv * qkv_bytes
    return decode_state_bytes(N, H, Dk, Dv) + N * H * per_head


def prefill_kernel_share_bytes(name: str, token_heads: int, num_seqs: int, H: int, Dk: int,
                               Dv: int, qkv_bytes: int, with_initial_state: bool,
                               with_final_state: bool) -> int | None:
    """The part of prefill_min_bytes that falls to one kernel of the two-kernel prefill: the
    chunk-local kernel reads every input once (q, k, v, log_alpha, beta); the state kernel writes
    o and reads / writes the fp32 states; the varlen chunk map reads cu_seqlens and writes the
    chunk offsets. The per-(chunk, head) records one kernel writes and the next reads are the split
    design's intermediates, not the method's work: they show up in measured traffic only."""
    states = num_seqs * H * Dk * Dv * 4
    if name.startswith("chunk_local"):
        return token_heads * ((2 * Dk + Dv) * qkv_bytes + 4 * Dk + 4)
    if name.startswith("chunk_state"):
        return token_heads * Dv * qkv_bytes + \
            states * (int(with_initial_state) + int(with_final_state))
    if name.startswith("chunk_map"):
        return 8 * (num_seqs + 1)
    return None
