"""Stage checks of the bf16 prefill: the chunk table of the plan kernel and the operator records of the
prep kernel, read back from the caller's workspace and compared with the fp64 oracle.

This is a white-box test. It restates the workspace layout of one prefill call (256-byte aligned
regions: meta int32[8], chunk offsets int32[N+1], the chunk table int4[nc_max], the segment table
int32[6N+1], the scan's sequence order int32[N], then one 25,088-byte operator record per (chunk,
head)) and the record format of the bf16 path. A record holds:
- [T''; P T''] as three bf16 parts of a 64 x 32 matrix in the 64-byte-swizzled K-major layout;
- the cross-chunk Gram G' = [K; Q] K_prev^T the same way;
- the gates Gamma_i, delta_i and Gamma_C.

Rows of a sequence's last chunk that lie beyond its end are padding. They carry the next tokens and
are never used, so only valid rows are compared.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_10_b200 import gdn
from linear_attention_10_b200.workloads import make_prefill_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
C = 32
RECORD = 25088
PART = 4096
CROSS = 3 * PART
GATE = 6 * PART


def _align(x):
    return (x + 255) & ~255


def _layout(T, N):
    nc_max = T // C + N
    o = 0
    off = {}
    off["meta"] = o
    o = _align(o + 8 * 4)
    off["chunk_off"] = o
    o = _align(o + (N + 1) * 4)
    off["chunk_tab"] = o
    o = _align(o + nc_max * 16)
    off["seg"] = o
    o = _align(o + (6 * N + 1) * 4)
    off["order"] = o
    o = _align(o + N * 4)
    off["op"] = o
    return off


def _sw64(r, k):
    return (r >> 3) * 512 + (r & 7) * 64 + (((k >> 3) ^ ((r >> 1) & 3)) << 4) + ((k & 7) << 1)


def _parts(rec, base, rows):
    """Sum of the three bf16 parts of a rows x 32 matrix stored at `base` of a record (fp64)."""
    r, k = np.indices((rows, C))
    off = _sw64(r, k)
    out = np.zeros((rows, C))
    for p in range(3):
        lo = rec[base + p * PART + off].astype(np.uint32)
        hi = rec[base + p * PART + off + 1].astype(np.uint32)
        bits = (lo | (hi << 8)) << 16
        out += bits.astype(np.uint32).view(np.float32).astype(np.float64)
    return out


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def test_plan_table_and_prep_records_match_the_oracle():
    lens = [70, 33, 0, 45]
    H, d = 2, 128
    inp = make_prefill_inputs(lens, H=H, dk=d, dv=d, dtype="bf16", seed=71, state_std=0.05, device=DEV)
    T, N = sum(lens), len(lens)
    ws = torch.zeros(gdn.workspace_bytes(T, N, H, d, d), dtype=torch.uint8, device=DEV)
    gdn.gdn_chunk_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], cu_seqlens=inp["cu_seqlens"],
                          state_in=inp["state_in"], workspace=ws)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_status() == 0
    w = ws.cpu().numpy()
    off = _layout(T, N)

    # plan stage: chunk count, per-sequence chunk offsets, and (sequence, first token, rows, -1) per chunk
    meta = w[off["meta"]:off["meta"] + 32].view(np.int32)
    counts = [(L + C - 1) // C for L in lens]
    assert meta[0] == sum(counts) and meta[1] == 0
    chunk_off = w[off["chunk_off"]:off["chunk_off"] + 4 * (N + 1)].view(np.int32)
    assert list(chunk_off) == list(np.concatenate([[0], np.cumsum(counts)]))
    tab = w[off["chunk_tab"]:off["chunk_tab"] + 16 * int(meta[0])].view(np.int32).reshape(-1, 4)
    expect = []
    t0 = 0
    for n, L in enumerate(lens):
        for c in range((L + C - 1) // C):
            expect.append([n, t0 + c * C, min(C, L - c * C), -1])
        t0 += L
    assert tab.tolist() == expect
    # the scan takes the sequences longest first (most chunks; ties by index)
    order = w[off["order"]:off["order"] + 4 * N].view(np.int32)
    assert list(order) == sorted(range(N), key=lambda n: (-counts[n], n))

    # prep stage: every (chunk, head) record against the oracle's chunk operator
    q, k = (inp[x].float().cpu().numpy().astype(np.float64) for x in ("q", "k"))
    g, b = (inp[x].cpu().numpy().astype(np.float64) for x in ("g", "beta"))
    for gc, (n, tc, L, _) in enumerate(expect):
        first = tc == sum(lens[:n])
        for h in range(H):
            rec = w[off["op"] + (gc * H + h) * RECORD:off["op"] + (gc * H + h + 1) * RECORD]
            rows = slice(tc, tc + L)
            kp = None if first else k[tc - C:tc, h]
            ref = oracle.chunk_operator(q[rows, h], k[rows, h], g[rows, h], b[rows, h], k_prev=kp)
            op = _parts(rec, 0, 2 * C)
            assert _rel(op[:C], ref["Tpp"]) < 1e-4, (gc, h, "T''")
            assert _rel(op[C:C + L], ref["PTpp"][:L]) < 1e-4, (gc, h, "P T''")
            if not first:
                gp = _parts(rec, CROSS, 2 * C)
                valid = np.r_[0:L, C:C + L]
                assert _rel(gp[valid], ref["Gp"][valid]) < 1e-4, (gc, h, "G'")
            gates = rec[GATE:GATE + 65 * 4].view(np.float32).astype(np.float64)
            assert _rel(gates[:C], ref["Gamma"]) < 1e-5
            assert _rel(gates[C:2 * C], ref["delta"]) < 1e-5
            assert abs(gates[2 * C] - ref["GammaC"]) <= 1e-5 * ref["GammaC"]
