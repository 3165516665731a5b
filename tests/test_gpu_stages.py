"""Stage checks of the bf16 prefill: the pair table of the plan kernel and the operator records of the
prep kernel, read back from the caller's workspace and compared with the fp64 oracle.

This is a white-box test. It restates the workspace layout of one prefill call (256-byte aligned
regions: meta int32[8], table offsets int32[N+1], the table int4[floor(T/32) + N], the segment table
int32[6N+1], the scan's sequence order int32[N], then one 49,664-byte operator record per (pair of
chunks, head)) and the record format of the bf16 path, which advances the state by 64 rows (two
chunks of 32) per step. A record holds:
- [T''; P T''] of the pair (128 x 64) as three bf16 parts in the 128-byte-swizzled K-major layout;
- the gates Gamma_i and delta_i of the pair's 64 rows.

The oracle's chunk operator over the pair's 64 rows is the reference: its T = (I + A)^-1 is what the
prep kernel forms from the two chunks' 32 x 32 inverses. Rows of a sequence's last pair that lie
beyond its end are padding. They carry the next tokens and are never used, so only the valid rows of
P T'' are compared.
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
PAIR = 64
RECORD = 49664
PART = 16384
GATE = 3 * PART


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


def _sw128(r, k):
    return (r >> 3) * 1024 + (r & 7) * 128 + (((k >> 3) ^ (r & 7)) << 4) + ((k & 7) << 1)


def _parts(rec, rows):
    """Sum of the three bf16 parts of a rows x 64 matrix at the start of a record (fp64)."""
    r, k = np.indices((rows, PAIR))
    off = _sw128(r, k)
    out = np.zeros((rows, PAIR))
    for p in range(3):
        lo = rec[p * PART + off].astype(np.uint32)
        hi = rec[p * PART + off + 1].astype(np.uint32)
        bits = (lo | (hi << 8)) << 16
        out += bits.astype(np.uint32).view(np.float32).astype(np.float64)
    return out


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def test_plan_table_and_prep_records_match_the_oracle():
    lens = [150, 33, 0, 45]
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

    # plan stage: pair count, per-sequence pair offsets, and (sequence, first token, rows, -1) per pair
    meta = w[off["meta"]:off["meta"] + 32].view(np.int32)
    counts = [(L + PAIR - 1) // PAIR for L in lens]
    assert meta[0] == sum(counts) and meta[1] == 0
    chunk_off = w[off["chunk_off"]:off["chunk_off"] + 4 * (N + 1)].view(np.int32)
    assert list(chunk_off) == list(np.concatenate([[0], np.cumsum(counts)]))
    tab = w[off["chunk_tab"]:off["chunk_tab"] + 16 * int(meta[0])].view(np.int32).reshape(-1, 4)
    expect = []
    t0 = 0
    for n, L in enumerate(lens):
        for c in range((L + PAIR - 1) // PAIR):
            expect.append([n, t0 + c * PAIR, min(PAIR, L - c * PAIR), -1])
        t0 += L
    assert tab.tolist() == expect
    # the scan takes the sequences longest first (most pairs; ties by index)
    order = w[off["order"]:off["order"] + 4 * N].view(np.int32)
    assert list(order) == sorted(range(N), key=lambda n: (-counts[n], n))

    # prep stage: every (pair, head) record against the oracle's operator over the pair's 64 rows
    q, k = (inp[x].float().cpu().numpy().astype(np.float64) for x in ("q", "k"))
    g, b = (inp[x].cpu().numpy().astype(np.float64) for x in ("g", "beta"))
    for gc, (n, tc, L, _) in enumerate(expect):
        for h in range(H):
            rec = w[off["op"] + (gc * H + h) * RECORD:off["op"] + (gc * H + h + 1) * RECORD]
            rows = slice(tc, tc + L)
            ref = oracle.chunk_operator(q[rows, h], k[rows, h], g[rows, h], b[rows, h], chunk=PAIR)
            op = _parts(rec, 2 * PAIR)
            assert _rel(op[:PAIR], ref["Tpp"]) < 1e-4, (gc, h, "T''")
            assert _rel(op[PAIR:PAIR + L], ref["PTpp"][:L]) < 1e-4, (gc, h, "P T''")
            gates = rec[GATE:GATE + 2 * PAIR * 4].view(np.float32).astype(np.float64)
            assert _rel(gates[:PAIR], ref["Gamma"]) < 1e-5
            assert _rel(gates[PAIR:], ref["delta"]) < 1e-5
