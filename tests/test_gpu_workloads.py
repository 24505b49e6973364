"""Full-size parity on the five workloads, in the launch configuration bench.py times.

The GPU runs the whole layer exactly as the benchmark step does:
seq_to_head(q, k, v) -> forward (fp32 O) -> head_to_seq(O); seq_to_head(dO)
-> backward (fp32) -> head_to_seq(dQ, dK, dV).  For b = 1 the seq-sharded
buffers are byte-identical to unsharded [n][H][d] tensors, so outputs are
indexed by (token, head) directly.

Compared against the fp64 oracle, element by element (tolerances as
everywhere: every element within 1e-2, sum|g-r|/sum|r| <= 2e-3 for
fp32-stored values, LSE max-abs <= 1e-3):
  * every element of O, LSE and dQ of all G query heads of one kv group and
    of that kv head's dK and dV, at full size (the Llama-8B shape, the packed
    SFT batch and the n = 131072 round trip; the oracle's per-head work runs
    in parallel processes);
  * O and LSE of sampled query rows of every head (rows 0 and n-1, the first
    and last row of random 128-row tiles, random rows), each against its
    full visible prefix;
  * dQ of sampled rows of every head;
  * dK and dV of the last W keys of every sample, for every kv head: only
    rows in [end - W, end) see them, so the oracle's row-window backward is
    exact there;
  * at every key, the column sums sum_j dK_j = 0 and sum_j dV_j = sum dO.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_util import LSE_MAX_ABS, assert_close, assert_lse_close, to_dev_bf16
from oracle_pool import heads_fwd_bwd

pytestmark = [pytest.mark.gpu, pytest.mark.large]

W_KEYS = 128


def sample_rows(rng, n, count):
    tiles = rng.integers(0, (n + 127) // 128, 4)
    rows = {0, n - 1}
    for t in tiles:
        rows.add(int(t) * 128)
        rows.add(min(n - 1, int(t) * 128 + 127))
    rows.update(int(r) for r in rng.integers(0, n, count))
    return np.array(sorted(rows))


def run_layer(w, x, dev, backward=True):
    """The benchmark step on device; returns host fp32 arrays in [n][H][d] form."""
    import ulysses_head_attention_b200 as uly
    P, n, hq, hkv, d = w.P, w.n, w.h_q, w.h_kv, w.d
    m = n // P

    def seq(bits):
        return to_dev_bf16(bits.reshape(P, 1, m, bits.shape[2], d), dev)

    q, k, v = seq(x["q"]), seq(x["k"]), seq(x["v"])
    pos = torch.from_numpy(x["position_ids"]).to(dev)
    head = {nm: torch.empty((P, 1, n, t.shape[3] // P, d), dtype=torch.bfloat16, device=dev)
            for nm, t in (("q", q), ("k", k), ("v", v))}
    for nm, t in (("q", q), ("k", k), ("v", v)):
        uly.ulysses_seq_to_head(t, head[nm])
    shape = uly.make_shape(1, n, hq, hkv, d, P)
    o_head = torch.empty((P, 1, n, hq // P, d), dtype=torch.float32, device=dev)
    lse = torch.empty((P, 1, hq // P, n), dtype=torch.float32, device=dev)
    ws_f = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(shape), dev)
    if w.rank_by_rank:
        for r in range(P):
            uly.ulysses_attn_fwd(head["q"], head["k"], head["v"], pos, o_head, lse, ws_f, rank=r)
    else:
        uly.ulysses_attn_fwd(head["q"], head["k"], head["v"], pos, o_head, lse, ws_f)
    o_seq = torch.empty((P, 1, m, hq, d), dtype=torch.float32, device=dev)
    uly.ulysses_head_to_seq(o_head, o_seq)
    assert uly.ulysses_workspace_status(ws_f) == 0
    out = {"o": o_seq.view(n, hq, d).cpu().numpy(),
           "lse": lse.view(P, hq // P, n).cpu().numpy().reshape(hq, n)}   # global head = r*hq/P + j
    del o_seq
    if backward:
        do = seq(x["do"])
        do_head = torch.empty_like(head["q"])
        uly.ulysses_seq_to_head(do, do_head)
        ws_b = uly.alloc_workspace(uly.ulysses_attn_bwd_workspace(shape, uly.ULY_F32), dev)
        g = {nm: torch.empty(head[nm].shape, dtype=torch.float32, device=dev) for nm in ("q", "k", "v")}
        uly.ulysses_attn_bwd(head["q"], head["k"], head["v"], o_head, lse, do_head, pos, g["q"], g["k"], g["v"], ws_b)
        assert uly.ulysses_workspace_status(ws_b) == 0
        for nm in ("q", "k", "v"):
            gs = torch.empty((P, 1, m, g[nm].shape[3] * P, d), dtype=torch.float32, device=dev)
            uly.ulysses_head_to_seq(g[nm], gs)
            out["d" + nm] = gs.view(n, -1, d).cpu().numpy()
    return out


def check_full_group(w, x, out, g):
    """Every element of one kv group: O, LSE, dQ of its G query heads and
    dK, dV of kv head g, against the oracle's blocked fp64 attention."""
    ss = oracle.segment_starts(x["position_ids"])[0]
    scale = oracle.default_scale(w.d)
    k = synthetic.bf16_bits_to_f64(x["k"][0, :, g])
    v = synthetic.bf16_bits_to_f64(x["v"][0, :, g])
    hs = list(range(g * w.group, (g + 1) * w.group))
    jobs = [(synthetic.bf16_bits_to_f64(x["q"][0, :, h]), k, v,
             synthetic.bf16_bits_to_f64(x["do"][0, :, h]) if w.backward else None, ss, scale) for h in hs]
    res = heads_fwd_bwd(jobs, backward=w.backward)
    what = f"{w.name} kv group {g} (all {w.group} query heads, every row)"
    assert_close(out["o"][:, hs], np.stack([r[0] for r in res], axis=1), f"{what} O")
    assert_lse_close(out["lse"][hs], np.stack([r[1] for r in res]), f"{what} LSE")
    if w.backward:
        assert_close(out["dq"][:, hs], np.stack([r[2] for r in res], axis=1), f"{what} dQ")
        assert_close(out["dk"][:, g], sum(r[3] for r in res), f"{w.name} kv head {g} dK (every key)")
        assert_close(out["dv"][:, g], sum(r[4] for r in res), f"{w.name} kv head {g} dV (every key)")


def check_forward(w, x, out, rng, rows_per_head):
    ss = oracle.segment_starts(x["position_ids"])[0]
    scale = oracle.default_scale(w.d)
    got, ref, gl, rl = [], [], [], []
    for g in range(w.h_kv):
        k = synthetic.bf16_bits_to_f64(x["k"][0, :, g])
        v = synthetic.bf16_bits_to_f64(x["v"][0, :, g])
        for h in range(g * w.group, (g + 1) * w.group):
            rows = sample_rows(rng, w.n, rows_per_head)
            q = synthetic.bf16_bits_to_f64(x["q"][0, :, h])
            o_r, l_r = oracle.attention_fwd_rows(q, k, v, ss, scale, rows)
            got.append(out["o"][rows, h]); ref.append(o_r)
            gl.append(out["lse"][h, rows]); rl.append(l_r)
    assert_close(np.concatenate(got), np.concatenate(ref), f"{w.name} O (sampled rows)")
    assert_lse_close(np.concatenate(gl), np.concatenate(rl), f"{w.name} LSE (sampled rows)")


def check_backward(w, x, out, rng, rows_per_head):
    ss = oracle.segment_starts(x["position_ids"])[0]
    scale = oracle.default_scale(w.d)
    ends = np.cumsum(x["lengths"][0])
    got_q, ref_q, got_kv, ref_kv = [], [], [], []
    for g in range(w.h_kv):
        k = synthetic.bf16_bits_to_f64(x["k"][0, :, g])
        v = synthetic.bf16_bits_to_f64(x["v"][0, :, g])
        dk_r = np.zeros_like(k)
        dv_r = np.zeros_like(v)
        keys = np.concatenate([np.arange(max(int(e) - W_KEYS, int(e) - int(L)), int(e))
                               for e, L in zip(ends, x["lengths"][0])])
        for h in range(g * w.group, (g + 1) * w.group):
            q = synthetic.bf16_bits_to_f64(x["q"][0, :, h])
            do = synthetic.bf16_bits_to_f64(x["do"][0, :, h])
            rows = sample_rows(rng, w.n, rows_per_head)
            got_q.append(out["dq"][rows, h])
            ref_q.append(oracle.attention_bwd_rows(q, k, v, do, ss, scale, rows))
            for e, L in zip(ends, x["lengths"][0]):
                lo = max(int(e) - W_KEYS, int(e) - int(L))
                _, a, b = oracle.attention_bwd_head(q, k, v, do, ss, scale, row_lo=lo, row_hi=int(e))
                dk_r[lo:e] += a[lo:e]
                dv_r[lo:e] += b[lo:e]
        got_kv.append(np.stack([out["dk"][keys, g], out["dv"][keys, g]]))
        ref_kv.append(np.stack([dk_r[keys], dv_r[keys]]))
        # column sums over every key of this kv head
        do_grp = synthetic.bf16_bits_to_f64(x["do"][0, :, g * w.group:(g + 1) * w.group]).sum(axis=(0, 1))
        dk_all = out["dk"][:, g].astype(np.float64)
        assert np.abs(dk_all.sum(axis=0)).max() <= 1e-3 * np.abs(dk_all).sum(axis=0).max()
        assert np.abs(out["dv"][:, g].astype(np.float64).sum(axis=0) - do_grp).max() <= 1e-3 * max(1.0, np.abs(do_grp).max())
    assert_close(np.concatenate(got_q), np.concatenate(ref_q), f"{w.name} dQ (sampled rows)")
    gk, rk = np.concatenate(got_kv, axis=1), np.concatenate(ref_kv, axis=1)
    assert_close(gk[0], rk[0], f"{w.name} dK (last {W_KEYS} keys of every sample)")
    assert_close(gk[1], rk[1], f"{w.name} dV (last {W_KEYS} keys of every sample)")


# kv group compared in full: the first rank's first group for the Llama-8B
# shape, the last rank's group for the packed batch
FULL_GROUP = {"llama8b_p4_n32k": 0, "packed_sft_p8_n64k": 7}


@pytest.mark.parametrize("name", ["tiny_p2_n256", "llama8b_p4_n32k", "packed_sft_p8_n64k", "roundtrip_p4_n128k"])
def test_workload_layer(cuda_device, name):
    w = synthetic.WORKLOADS[name]
    x = synthetic.make_inputs(w)
    out = run_layer(w, x, cuda_device, backward=w.backward)
    rng = np.random.default_rng(w.wid)
    if name == "tiny_p2_n256":
        # small enough for the full layer in the oracle
        qs, ks, vs = (oracle.shard(synthetic.bf16_bits_to_f64(x[t]), w.P) for t in ("q", "k", "v"))
        O_ref, L_ref = oracle.ulysses_layer_fwd(qs, ks, vs, x["position_ids"], w.P)
        assert_close(out["o"], oracle.unshard(O_ref)[0], "tiny O (all elements)")
        assert np.abs(out["lse"] - L_ref.transpose(1, 0, 2, 3).reshape(w.h_q, w.n)).max() <= LSE_MAX_ABS
        return
    if name in FULL_GROUP:
        check_full_group(w, x, out, FULL_GROUP[name])
    check_forward(w, x, out, rng, rows_per_head=24)
    if w.backward:
        check_backward(w, x, out, rng, rows_per_head=12)


@pytest.mark.oracle_heavy
def test_roundtrip_full_kv_group_0(cuda_device):
    """The full layer round trip at n = 131072: every element of O, LSE, dQ of
    kv group 0's four query heads and of kv head 0's dK, dV against the
    oracle (about 5e13 flops of fp64 on the host, spread over its cores)."""
    w = synthetic.WORKLOADS["roundtrip_p4_n128k"]
    x = synthetic.make_inputs(w)
    out = run_layer(w, x, cuda_device, backward=True)
    check_full_group(w, x, out, 0)


def test_workload_long_context_rank_by_rank(cuda_device):
    """n = 524288, each virtual rank's 4-head slice computed in turn."""
    w = synthetic.WORKLOADS["long_p8_n512k"]
    x = synthetic.make_inputs(w, with_do=False)
    out = run_layer(w, x, cuda_device, backward=False)
    check_forward(w, x, out, np.random.default_rng(w.wid), rows_per_head=6)
