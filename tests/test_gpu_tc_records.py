"""The bf16 tensor-core path's per-chunk records, decoded from the workspace and checked against the
chunk formulas of "Kimi Linear: An Expressive, Efficient Attention Architecture" (paper-graph-ui
walkthrough, §3.4 "Chunkwise Parallelization") evaluated here in fp64 from the same inputs.

This localises a failure of the end-to-end parity tests to the chunk-local kernel (records wrong)
or to the state kernel (records right, outputs wrong). Record layout per (chunk, head), bf16
tiles in the 128-byte-swizzled operand layout: [Qt; W] [128 x 128], Kt [64 x 128], A_qk [64 x 64],
U [64 x 128],
then gamma_C as 128 fp32. Qt and W share one [128 x 128] tile (Qt rows 0..63, W rows 64..127).
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_120_b200 as kda
import kda_synth
from kda_synth import PrefillSpec
from tests._parity import to_np

pytestmark = pytest.mark.gpu

REC = dict(QW=0, Kt=32768, Aqk=49152, U=57344, gam=73728, size=74240)


def tile_index(rows, cols):
    """Element offsets (in bf16 units) of a [rows x cols] tile in the swizzled operand layout."""
    r = np.arange(rows)[:, None]
    c = np.arange(cols)[None, :]
    block = rows * 128
    off = (c // 64) * block + (r // 8) * 1024 + (r % 8) * 128 + (((c % 64) // 8) ^ (r % 8)) * 16 \
        + (c % 8) * 2
    return off // 2


def decode_tile(buf_u8: np.ndarray, base: int, rows: int, cols: int) -> np.ndarray:
    bf = buf_u8[base:base + rows * cols * 2].view(np.uint16).astype(np.uint32) << 16
    vals = bf.view(np.float32)
    return vals[tile_index(rows, cols)].astype(np.float64)


def chunk_reference(k, q, v, la, beta, L):
    """fp64 W, Qt, Kt, A_qk, U, gamma_C of one chunk (rows >= L are identity padding)."""
    C = 64
    K = np.zeros((C, 128)); Q = np.zeros((C, 128)); V = np.zeros((C, 128))
    G = np.zeros((C, 128)); b = np.zeros(C)
    K[:L], Q[:L], V[:L], G[:L], b[:L] = k, q, v, la, beta
    g = np.cumsum(G, axis=0)
    # [r, i, c] = gamma_r / gamma_i on the causal pairs i <= r (exponent <= 0), 0 elsewhere: the
    # mask is applied before the exponential, so no masked pair overflows and a NaN would show
    causal = np.arange(C)[:, None, None] >= np.arange(C)[None, :, None]
    ratio = np.zeros((C, C, 128))
    np.exp(g[:, None, :] - g[None, :, :], out=ratio, where=np.broadcast_to(causal, ratio.shape))
    akk = np.einsum("rc,ic,ric->ri", K, K, ratio)
    aqk = np.einsum("rc,ic,ric->ri", Q, K, ratio)
    A = np.tril(b[:, None] * akk, -1)
    M = np.linalg.inv(np.eye(C) + A) * b[None, :]
    W = M @ (np.exp(g) * K)
    U = M @ V
    return dict(W=W, Qt=np.exp(g) * Q, Kt=np.exp(g[-1] - g) * K, Aqk=np.tril(aqk), U=U,
                gam=np.exp(g[-1]))


def chunk_mode(la_chunk: np.ndarray, limit: float = 60.0, shifted: bool = False) -> str:
    """Which evaluation of A_kk / A_qk the kernel picks for one chunk of one head: "fast" when
    every channel decays by at most exp(-limit) over the chunk; with `shifted` (the kernel built
    for the in-kernel gate) "shifted" — the fast evaluation around a per-channel reference at
    half the channel's decay — when every channel decays by at most exp(-2 limit); "blocks" when
    every channel decays by at most exp(-limit) within every 16-row block; "exact" otherwise. The
    limit is 60 for caller-provided keys and 80 when the kernel L2-normalises them."""
    g = np.concatenate([np.zeros((1, la_chunk.shape[1])), np.cumsum(la_chunk, axis=0)])
    if g[-1].min() >= -limit:
        return "fast"
    if shifted and g[-1].min() >= -2 * limit:
        return "shifted"
    ends = [min(16 * (R + 1), la_chunk.shape[0]) for R in range(4)]
    starts = [min(16 * R, la_chunk.shape[0]) for R in range(4)]
    drops = [(g[s] - g[e]).max() for s, e in zip(starts, ends)]
    return "blocks" if max(drops) <= limit else "exact"


# per-chunk decays: (channels, per-token level or None for the plain recipe, scale). A level
# replaces the channels' log decays by level + 0.05 x the plain ones (a small per-token spread):
# -1.4 decays a channel by 90-97 nats over a chunk (between 60 and 120), -2.2 by 141-148 nats
# (beyond 120) but 35-37 nats per 16-row block (within 60).
MIXED_MODES = [(slice(None), None, 1.0), (slice(None), -1.4, 1.0), (slice(None), -2.2, 1.0),
               (slice(None), None, 40.0), (slice(0, 32), -2.2, 1.0)]


@pytest.mark.parametrize("T,mixed,gate", [(64, False, "given"), (150, False, "given"),
                                          (314, True, "given"), (314, True, "in_kernel")])
def test_chunk_records_match_formulas(cuda_device, T, mixed, gate):
    spec = PrefillSpec("t", B=1, T=T, H=2, Dk=128, Dv=128, chunk=64, dtype="bf16", decay="fast",
                       init_std=0.02)
    inp = kda_synth.prefill_inputs(spec, 500 + T, cuda_device)
    in_kernel = gate == "in_kernel"
    if mixed:  # one chunk in each mode, the block mode twice (all channels / 32 of them, ragged)
        la = inp["log_alpha"].clone()
        for c, (chs, level, f) in enumerate(MIXED_MODES):
            part = la[:, 64 * c:64 * c + 64, :, chs]
            la[:, 64 * c:64 * c + 64, :, chs] = f * part if level is None else level + 0.05 * part
        inp["log_alpha"] = la
        modes = [chunk_mode(to_np(la[0, 64 * c:64 * c + 64, h]), shifted=in_kernel)
                 for c in range(5) for h in range(2)]
        assert modes == (["fast"] * 2 + ["shifted" if in_kernel else "blocks"] * 2 +
                         ["blocks"] * 2 + ["exact"] * 2 + ["blocks"] * 2), modes
    fusion, la_in = None, inp["log_alpha"]
    if in_kernel:
        # the kernel forms log alpha = -exp(A_log) softplus(g + dt_bias); with A_log = 0 and
        # dt_bias = 0 the raw gate g = log(expm1(-log alpha)) gives back the decays above, and
        # the formulas take -softplus(g) of the fp32 g the kernel reads
        y = (-inp["log_alpha"].double()).clamp_min(1e-6)
        la_in = torch.log(torch.expm1(y)).float()
        inp["log_alpha"] = -torch.nn.functional.softplus(la_in.double())
        fusion = dict(A_log=torch.zeros((2,), device=cuda_device),
                      dt_bias=torch.zeros((2, 128), device=cuda_device))
    nbytes = kda.kda_chunk_fwd_workspace_size(1, T, 2, 128, 128, 64, 1, torch.bfloat16)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=cuda_device)
    kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], la_in, inp["beta"],
                      initial_state=inp["initial_state"], chunk=64, workspace=ws, fusion=fusion)
    torch.cuda.synchronize()
    assert kda.kda_last_device_error() == kda.KDA_OK
    buf = ws.cpu().numpy()
    x = {n: to_np(inp[n][0]) for n in ("q", "k", "v", "log_alpha", "beta")}
    nchunks = (T + 63) // 64
    for c in range(nchunks):
        t0 = 64 * c
        L = min(64, T - t0)
        for h in range(2):
            ref = chunk_reference(x["k"][t0:t0 + L, h], x["q"][t0:t0 + L, h],
                                  x["v"][t0:t0 + L, h], x["log_alpha"][t0:t0 + L, h],
                                  x["beta"][t0:t0 + L, h], L)
            base = 256 + REC["size"] * (c * 2 + h)
            qw = decode_tile(buf, base + REC["QW"], 128, 128)
            got = dict(W=qw[64:], Qt=qw[:64],
                       Kt=decode_tile(buf, base + REC["Kt"], 64, 128),
                       Aqk=decode_tile(buf, base + REC["Aqk"], 64, 64),
                       U=decode_tile(buf, base + REC["U"], 64, 128),
                       gam=buf[base + REC["gam"]:base + REC["gam"] + 512].view(np.float32))
            for name in ("Qt", "Kt", "Aqk", "W", "U", "gam"):
                r, gval = ref[name], np.asarray(got[name], dtype=np.float64)
                err = np.abs(gval - r).max() / max(np.abs(r).max(), 1e-30)
                assert err <= 2e-2, f"chunk {c} head {h} {name}: rel err {err:.3e}"
