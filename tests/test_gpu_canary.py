"""Guard regions around every output of the three calls (needs a B200).

The header promises that each call writes only inside its outputs: `out`
only at the N valid tokens of each head (there is no padded row in the
[B,H,N,D] layout, and padded block positions are skipped by the TMA stores),
`kv_idx` only in the first kv_cnt entries of each row, the schedule's `work`
only in its first B*H*units entries. Each output here sits inside a larger
buffer whose guard regions, and unused row tails, hold a sentinel that no
call writes; after route, schedule and attention the sentinels must all be
intact and every valid output element overwritten.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_fvattn_b200 import inputs as gen
from tests import fvtest

pytestmark = pytest.mark.gpu

GUARD = 4096                     # elements on each side (keeps 16-byte alignment)
SENT_I32 = -0x5A5A5A5B
SENT_F32_BITS = 0x7FBADBAD       # a NaN payload no kernel produces
SENT_16 = 0x7FC3                 # a bf16/fp16 NaN payload no kernel produces


def _signed(bits, width):
    return bits - (1 << width) if bits >= 1 << (width - 1) else bits


def _guarded(shape, dtype, sentinel_bits):
    """A buffer of the output's size plus GUARD elements on each side, all set
    to the sentinel; returns (the raw integer view, the output view)."""
    n = int(np.prod(shape))
    if dtype in (torch.bfloat16, torch.float16):
        raw = torch.full((n + 2 * GUARD,), _signed(sentinel_bits, 16), dtype=torch.int16, device="cuda")
        buf = raw.view(dtype)
    elif dtype == torch.float32:
        raw = torch.full((n + 2 * GUARD,), _signed(sentinel_bits, 32), dtype=torch.int32, device="cuda")
        buf = raw.view(torch.float32)
    else:
        raw = torch.full((n + 2 * GUARD,), sentinel_bits, dtype=dtype, device="cuda")
        buf = raw
    return raw, buf[GUARD:GUARD + n].view(shape)


def _guards_intact(raw, sentinel):
    r = raw.cpu().numpy()
    return bool((r[:GUARD] == sentinel).all() and (r[-GUARD:] == sentinel).all())


CASES = [
    gen.custom("canary_ragged", 1, 3, 128, (9, 20, 28), (4, 8, 8), 0.9, 4, sigma=2.0, a_range=(0.5, 4.0), seed=61),
    gen.custom("canary_64tok_odd", 2, 2, 128, (4, 12, 20), (4, 4, 4), 0.8, 2, sigma=1.5, a_range=(0.5, 4.0),
               seed=62),
    gen.custom("canary_d64_ragged", 1, 2, 64, (6, 10, 9), (4, 4, 4), 0.9, 3, sigma=1.5, a_range=(0.5, 4.0), seed=63),
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_outputs_write_nothing_outside_their_extent(wl):
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    q, k, v = fvtest.make_on_gpu(wl)
    geo = fvtest.geometry(wl)
    nb = fa.num_blocks(geo)
    C = 148
    BH = wl.B * wl.H
    units = -(-nb // 4) if wl.block[0] * wl.block[1] * wl.block[2] == 64 else nb
    ws = torch.zeros(fa.workspace_size(geo, C), dtype=torch.uint8, device="cuda")
    fa.workspace_init(ws)
    s16 = _signed(SENT_16, 16)
    s32f = _signed(SENT_F32_BITS, 32)
    raw_cnt, cnt = _guarded((wl.B, wl.H, nb), torch.int32, SENT_I32)
    raw_idx, idx = _guarded((wl.B, wl.H, nb, nb), torch.int32, SENT_I32)
    raw_prob, probs = _guarded((wl.B, wl.H, nb, nb), torch.float32, SENT_F32_BITS)
    raw_work, work = _guarded((BH * nb,), torch.int32, SENT_I32)
    raw_rng, rng = _guarded((C + 1,), torch.int32, SENT_I32)
    raw_cost, cost = _guarded((C,), torch.int64, SENT_I32)
    raw_ns, ns = _guarded((C,), torch.int64, SENT_I32)
    raw_out, out = _guarded(tuple(q.shape), q.dtype, SENT_16)

    fa.route(geo, q, k, wl.p, wl.k_min, cnt, idx, ws, probs)
    fa.schedule(geo, cnt, idx, False, C, work, rng, ws, cost)
    fa.sparse_attn(geo, q, k, v, cnt, idx, work, rng, C, False, out, ws, ns)
    torch.cuda.synchronize()
    assert fa.read_device_status(ws) == 0

    for raw, sent in ((raw_cnt, SENT_I32), (raw_idx, SENT_I32), (raw_prob, s32f), (raw_work, SENT_I32),
                      (raw_rng, SENT_I32), (raw_cost, SENT_I32), (raw_ns, SENT_I32), (raw_out, s16)):
        assert _guards_intact(raw, sent)
    c = cnt.cpu().numpy()
    ix = idx.cpu().numpy()
    assert ((c >= 1) & (c <= nb)).all()
    tail = np.arange(nb)[None, None, None, :] >= c[..., None]
    assert (ix[tail] == SENT_I32).all(), "kv_idx written past kv_cnt"
    assert (ix[~tail] != SENT_I32).all()
    w = work.cpu().numpy()
    U = int(rng[C].item())          # units of the schedule (long 64-token units may run split)
    assert U >= BH * units
    assert (w[U:] == SENT_I32).all(), "work written past the unit count"
    assert len(set(w[:U].tolist())) == U
    assert not torch.isnan(probs).any()
    o = out.view(torch.int16).cpu().numpy()
    assert (o != s16).all(), "a valid output element was left unwritten"
    assert torch.isfinite(out).all()
