"""hca_cache_append / hca_decode_step vs the fp64 oracle.

Sequences start at lengths on both sides of block boundaries and take ten
serving steps (one new token each per step).  After the steps the raw rings
must equal the newest tokens exactly (a copy), every compressed entry must
match the oracle's whole-sequence compression within the cache tolerance,
and the decode output of the last step (through hca_decode_step) must match
the oracle's decode on the oracle's cache."""
import numpy as np
import pytest
import torch

import compressed_sliding_window_b200 as hca
from compressed_sliding_window_b200 import inputs as I
from oracle import hca_oracle as O
from tests.gpu_util import assert_close_cache, assert_close_out, need_gpu, to64

pytestmark = pytest.mark.gpu

STEPS = 10


def _ring(x: torch.Tensor, L: int) -> torch.Tensor:
    return I.ring_window(x if x.dim() == 2 else x[:, None], L)


def _sequences(L0s, seed):
    cfg = I.DecodeConfig("append", S=len(L0s), seed=seed, ctx=1)
    return [I.decode_raw_sequence(cfg, i, L0 + STEPS) for i, L0 in enumerate(L0s)]


def _initial_state(raw, L0s, max_nc):
    S = len(L0s)
    ck = torch.zeros((S, max_nc, 512), dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros_like(ck)
    wk = torch.zeros((S, 128, 512), dtype=torch.bfloat16)
    wv = torch.zeros_like(wk)
    ws = torch.zeros((S, 128), dtype=torch.bfloat16)
    for i, ((k, v, s), L0) in enumerate(zip(raw, L0s)):
        nb = L0 // 128
        if nb:
            e_k, e_v = hca.compress(k[None, :L0].cuda(), v[None, :L0].cuda(), s[None, :L0].cuda())
            ck[i, :nb] = e_k[0]
            cv[i, :nb] = e_v[0]
        wk[i] = _ring(k, L0)
        wv[i] = _ring(v, L0)
        ws[i] = _ring(s, L0)[:, 0]
    return ck, cv, wk.cuda(), wv.cuda(), ws.cuda()


def test_append_steps_match_oracle():
    need_gpu()
    L0s = [1, 120, 127, 250, 1020, 4090]
    raw = _sequences(L0s, seed=61)
    max_nc = max((L0 + STEPS) // 128 for L0 in L0s)
    ck, cv, wk, wv, ws = _initial_state(raw, L0s, max_nc)
    S = len(L0s)
    cfg = I.DecodeConfig("append_q", S=S, seed=62, ctx=1)
    q, g = (t.cuda() for t in I.decode_query(cfg))
    out = None
    for step in range(STEPS):
        lens = [L0 + step + 1 for L0 in L0s]
        ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
        k_new = torch.stack([k[L - 1] for (k, _, _), L in zip(raw, lens)]).cuda()
        v_new = torch.stack([v[L - 1] for (_, v, _), L in zip(raw, lens)]).cuda()
        s_new = torch.stack([s[L - 1] for (_, _, s), L in zip(raw, lens)]).cuda()
        if step < STEPS - 1:
            hca.cache_append(k_new, v_new, s_new, ctx, wk, wv, ws, ck, cv)
        else:
            out = hca.decode_step(q, g, k_new, v_new, s_new, ctx, wk, wv, ws, ck, cv)
    torch.cuda.synchronize()
    code, where = hca.device_error()
    assert code == 0, f"device error {code} at {where}"
    lens = [L0 + STEPS for L0 in L0s]
    ref_ck = np.zeros((S, max_nc, 512))
    ref_cv = np.zeros((S, max_nc, 512))
    for i, ((k, v, s), L) in enumerate(zip(raw, lens)):
        # the rings hold copies of the newest tokens: bit-exact
        assert torch.equal(wk[i].cpu(), _ring(k, L)), f"wk seq {i}"
        assert torch.equal(wv[i].cpu(), _ring(v, L)), f"wv seq {i}"
        assert torch.equal(ws[i].cpu(), _ring(s, L)[:, 0]), f"ws seq {i}"
        nb = L // 128
        if nb:
            rck, rcv = O.compress(to64(k[None, :L]), to64(v[None, :L]), to64(s[None, :L]))
            assert_close_cache(to64(ck[i, :nb]), rck[0], f"ck seq {i}")
            assert_close_cache(to64(cv[i, :nb]), rcv[0], f"cv seq {i}")
            ref_ck[i, :nb], ref_cv[i, :nb] = rck[0], rcv[0]
    ref = O.decode_forward(to64(q), ref_ck, ref_cv, to64(wk), to64(wv), lens, to64(g))
    assert_close_out(to64(out), ref, "decode after append")


def test_append_reports_entry_beyond_capacity():
    """A block that completes past max_nc writes no entry and is reported as a
    device-side input error (nothing faults)."""
    need_gpu()
    S = 2
    k_new = torch.ones((S, 512), dtype=torch.bfloat16, device="cuda")
    s_new = torch.zeros((S,), dtype=torch.bfloat16, device="cuda")
    wk = torch.zeros((S, 128, 512), dtype=torch.bfloat16, device="cuda")
    wv, ws = torch.zeros_like(wk), torch.zeros((S, 128), dtype=torch.bfloat16, device="cuda")
    ck = torch.zeros((S, 1, 512), dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros_like(ck)
    ctx = torch.tensor([128, 256], dtype=torch.int32, device="cuda")   # entries 0 and 1
    hca.cache_append(k_new, k_new, s_new, ctx, wk, wv, ws, ck, cv)
    code, _ = hca.device_error()
    assert code == 5   # HCA_ERR_DEVICE_INPUT: entry 1 does not fit
    assert hca.device_error()[0] == 0
    # sequence 0's entry 0 was written; sequence 1 got none
    assert float(ck[1].float().abs().max()) == 0.0
    assert float(ck[0].float().abs().max()) > 0.0
