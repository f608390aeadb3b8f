"""Pins for the backward oracle (no GPU).

``oracle.backward`` is checked against things other than itself:

* central finite differences of the (separately pinned) forward oracle for
  the loss L = sum(dout * out), in float64;
* torch float64 autograd of an independent dense-mask restatement of the
  forward (masks built here with plain loops from idx / window, softmax with
  the sink as an extra column, as "Support attn sink in fa3", pull request
  1415, describes the sink);
* closed forms: a one-key window reduces the softmax to a logistic function
  of (s - sink) whose derivative is p (1 - p); the value-gradient column sum
  equals sum (1 - p_sink) dout because the key probabilities of a row sum to
  1 - p_sink;
* the full-coverage / wide-window equalities with dense causal attention
  ("Unified sparse attention API (dispatcher)" page, model-config key points).

The backward itself is read as the exact gradient of the forward of
"HySparse MQA sparse attention (FA4 block scoring + SWA MQA + block-sparse
DSA gather)", PaddleFleet pull request 1470 ("Core" list: SWA and block-sparse
MQA with backward passes, analytic attn_sink gradient).
"""

import math

import numpy as np
import pytest
import torch

import oracle.backward as OB
import oracle.hysparse as O
from block_sparse_mqa_b200 import synth


def _np(x):
    return x.detach().cpu().double().numpy()


def _case(T, H, dk, dv, docs, seed):
    inp = synth.make_inputs(T, H, dk, dv, dtype=torch.float32, seed=seed, doc_lengths=docs)
    rng = np.random.default_rng(seed + 100)
    dout = rng.standard_normal((T, H, dv))
    return _np(inp.q), _np(inp.k), _np(inp.v), _np(inp.sink), inp.cu_seqlens.tolist(), dout


def _idx(q, k, cu, B, K):
    bs = O.block_score(q, k, cu, B)
    return O.select_topk(bs["block_score"], cu, B, K)


# ---------------------------------------------------------------------------
# independent dense-mask restatement (plain loops for the key sets)
# ---------------------------------------------------------------------------

def _mask_sparse(T, cu, idx, B):
    m = np.zeros((T, T), dtype=bool)
    for d in range(len(cu) - 1):
        bos, eos = cu[d], cu[d + 1]
        for t in range(bos, eos):
            bq = (t - bos) // B
            row = [int(x) for x in idx[t]]
            for s, b in enumerate(row):
                # used when in [0, bq] and above the raw entry before it
                if b < 0 or b > bq or (s > 0 and b <= row[s - 1]):
                    continue
                for j in range(bos + b * B, min(bos + (b + 1) * B, eos)):
                    if j <= t:
                        m[t, j] = True
    return m


def _mask_window(T, cu, W):
    m = np.zeros((T, T), dtype=bool)
    for d in range(len(cu) - 1):
        bos, eos = cu[d], cu[d + 1]
        for t in range(bos, eos):
            for j in range(max(bos, t - W + 1), t + 1):
                m[t, j] = True
    return m


def _torch_grads(q, k, v, sink, dout, mask, scale):
    qt = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    kt = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    vt = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    st = torch.tensor(sink, dtype=torch.float64, requires_grad=True) if sink is not None else None
    T, H, _ = q.shape
    logits = scale * torch.einsum("thd,jd->thj", qt, kt)
    logits = logits.masked_fill(~torch.tensor(mask)[:, None, :], float("-inf"))
    if st is not None:
        logits = torch.cat([logits, st.view(1, H, 1).expand(T, H, 1)], dim=2)
    p = torch.softmax(logits, dim=2)[:, :, :T]
    out = torch.einsum("thj,je->the", p, vt)
    (out * torch.tensor(dout)).sum().backward()
    return (qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy(),
            st.grad.numpy() if st is not None else None)


@pytest.mark.parametrize("with_sink", [True, False])
@pytest.mark.parametrize("kind", ["sparse", "swa"])
def test_backward_matches_torch_autograd(kind, with_sink):
    docs = [23, 9, 32]
    T = sum(docs)
    q, k, v, sink, cu, dout = _case(T, 4, 24, 20, docs, seed=3)
    sink = sink if with_sink else None
    sc = 24 ** -0.5
    if kind == "sparse":
        B, K = 4, 3
        idx = _idx(q, k, cu, B, K)
        if with_sink:  # a row without a usable block: only the sink is left
            idx[30] = -1
        g = OB.sparse_mqa_bwd(q, k, v, dout, idx, cu, B, sink=sink)
        mask = _mask_sparse(T, cu, idx, B)
    else:
        W = 6
        g = OB.swa_mqa_bwd(q, k, v, dout, cu, W, sink=sink)
        mask = _mask_window(T, cu, W)
    tq, tk, tv, ts = _torch_grads(q, k, v, sink, dout, mask, sc)
    np.testing.assert_allclose(g["dq"], tq, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dk"], tk, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dv"], tv, rtol=1e-10, atol=1e-12)
    if with_sink:
        np.testing.assert_allclose(g["dsink"], ts, rtol=1e-10, atol=1e-12)
    else:
        assert g["dsink"] is None


def test_backward_matches_finite_differences():
    docs = [11, 7]
    T = sum(docs)
    q, k, v, sink, cu, dout = _case(T, 2, 8, 6, docs, seed=5)
    B, K = 4, 2
    idx = _idx(q, k, cu, B, K)
    g = OB.sparse_mqa_bwd(q, k, v, dout, idx, cu, B, sink=sink)

    def loss(q_, k_, v_, s_):
        return float((O.sparse_mqa_fwd(q_, k_, v_, idx, cu, B, sink=s_)["out"] * dout).sum())

    eps = 1e-6
    rng = np.random.default_rng(0)
    for name, arr, pos in (("dq", q, 0), ("dk", k, 1), ("dv", v, 2), ("dsink", sink, 3)):
        for _ in range(6):
            flat = rng.integers(arr.size)
            args = [q, k, v, sink]
            hi = [a.copy() for a in args]
            lo = [a.copy() for a in args]
            hi[pos].reshape(-1)[flat] += eps
            lo[pos].reshape(-1)[flat] -= eps
            fd = (loss(*hi) - loss(*lo)) / (2 * eps)
            an = g[name].reshape(-1)[flat]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, flat, fd, an)


def test_one_key_window_logistic_closed_form():
    # W = 1: each query attends only itself; p = 1 / (1 + exp(sink - s)),
    # out = p v_t, so d out / d s = p (1 - p) v_t and d out / d sink = -p (1 - p) v_t.
    T, H, dk, dv = 10, 3, 16, 12
    q, k, v, sink, cu, dout = _case(T, H, dk, dv, [T], seed=9)
    sc = dk ** -0.5
    g = OB.swa_mqa_bwd(q, k, v, dout, cu, 1, sink=sink)
    for t in range(T):
        for h in range(H):
            s = sc * float(q[t, h] @ k[t])
            p = 1.0 / (1.0 + math.exp(sink[h] - s))
            g_s = p * (1 - p) * float(dout[t, h] @ v[t])
            np.testing.assert_allclose(g["dq"][t, h], sc * g_s * k[t], rtol=1e-11, atol=1e-13)
    ddsink = np.zeros(H)
    dvv = np.zeros((T, dv))
    for t in range(T):
        for h in range(H):
            s = sc * float(q[t, h] @ k[t])
            p = 1.0 / (1.0 + math.exp(sink[h] - s))
            ddsink[h] += -p * (1 - p) * float(dout[t, h] @ v[t])
            dvv[t] += p * dout[t, h]
    np.testing.assert_allclose(g["dsink"], ddsink, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(g["dv"], dvv, rtol=1e-11, atol=1e-13)


def test_value_gradient_column_sum():
    docs = [40, 24]
    T = sum(docs)
    q, k, v, sink, cu, dout = _case(T, 4, 16, 8, docs, seed=11)
    B, K = 8, 3
    idx = _idx(q, k, cu, B, K)
    g = OB.sparse_mqa_bwd(q, k, v, dout, idx, cu, B, sink=sink)
    lse = O.sparse_mqa_fwd(q, k, v, idx, cu, B, sink=sink)["lse"]
    psink = np.exp(sink[None, :] - lse)                         # [T, H]
    expect = ((1.0 - psink)[:, :, None] * dout).sum(axis=(0, 1))
    np.testing.assert_allclose(g["dv"].sum(axis=0), expect, rtol=1e-10, atol=1e-10)
    # dsink is minus the sink probability times delta, summed over tokens
    out = O.sparse_mqa_fwd(q, k, v, idx, cu, B, sink=sink)["out"]
    delta = (dout * out).sum(axis=2)
    np.testing.assert_allclose(g["dsink"], -(psink * delta).sum(axis=0), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["delta"], delta, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("docs", [[37], [20, 17, 5]])
def test_full_coverage_and_wide_window_equal_dense(docs):
    T = sum(docs)
    q, k, v, sink, cu, dout = _case(T, 2, 16, 8, docs, seed=13)
    B = 8
    nb = max(O.num_blocks(e - b, B) for b, e in O.doc_bounds(cu))
    idx = np.full((T, nb), -1, dtype=np.int64)
    for b0, e0 in O.doc_bounds(cu):
        for t in range(b0, e0):
            n = (t - b0) // B + 1
            idx[t, :n] = np.arange(n)
    dense = OB.dense_causal_bwd(q, k, v, dout, cu, sink=sink)
    sp = OB.sparse_mqa_bwd(q, k, v, dout, idx, cu, B, sink=sink)
    sw = OB.swa_mqa_bwd(q, k, v, dout, cu, T + 3, sink=sink)
    for key in ("dq", "dk", "dv", "dsink"):
        np.testing.assert_array_equal(sp[key], dense[key])
        np.testing.assert_array_equal(sw[key], dense[key])
