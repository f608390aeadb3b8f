"""Plain float64 CPU definition of the backward of the block-sparse and
sliding-window MQA attention steps.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module;
only ``tests/`` call it.  It shares no code with the CUDA library.

Sources (web pages, cited by title and section):

* [HS] "HySparse MQA sparse attention (FA4 block scoring + SWA MQA +
  block-sparse DSA gather)", PaddleFleet pull request 1470: the "Core" list
  (the SWA and block-sparse MQA kernels come with backward passes; the
  learnable per-head attn_sink has an analytic gradient) and the Copilot
  per-file table (``windowed_mqa_attn*.py``: fwd/bwd with Dk != Dv,
  attn_sink and a guard for ragged sequence lengths in the backward;
  ``block_sparse_mqa_dsa.py``: analytic sink gradient).
* [SINK] "Support attn sink in fa3", PaddleFleet pull request 1415: the sink
  is a softmax offset (an extra logit in the denominator, no value row).

The pages give no formulas for the backward.  Reading taken: the backward is
the exact gradient of the forward defined in ``oracle.hysparse`` (the lse
includes the sink) for a scalar loss whose gradient with respect to ``out``
is ``dout``.  Per query token t with key set S_t, head h, s_j = scale *
<q[t,h], k[j]>, p_j = exp(s_j - lse), p_sink = exp(sink_h - lse):

    dp_j   = <dout[t,h], v[j]>
    delta  = <dout[t,h], out[t,h]>            (= sum_j p_j dp_j)
    ds_j   = p_j (dp_j - delta)
    dq[t,h]  = scale * sum_j ds_j k[j]
    dk[j]   += scale * ds_j q[t,h]            (summed over every (t, h))
    dv[j]   += p_j dout[t,h]                  (summed over every (t, h))
    dsink_h += -p_sink * delta                (summed over t)

The sink row follows from out depending on sink_h only through lse, and
d lse / d sink_h = p_sink.  A token with an empty key set (an idx row without
a usable block) has out = 0, lse = sink and contributes no gradient.  All
arithmetic is float64; sums over keys and heads are matrix products of the
library routine (numpy), sums over tokens run in ascending token order.
"""

from __future__ import annotations

from typing import Optional

import numpy as np

from .hysparse import (_f64, _scale, doc_bounds, sparse_key_set, window_key_set)

__all__ = ["attend_bwd", "sparse_mqa_bwd", "swa_mqa_bwd", "dense_causal_bwd"]


def attend_bwd(q_t, keys, k, v, sink, scale: float, dout_t):
    """Backward of one query token's H heads over ``keys`` ([HS] "Core";
    formulas in the module docstring).  Returns
    (dq_t [H, Dk], dk_part [n, Dk], dv_part [n, Dv], dsink_part [H],
    delta [H], out [H, Dv], lse [H]); the parts are this token's
    contributions to the listed keys."""
    q_t = _f64(q_t)
    H = q_t.shape[0]
    kk = _f64(k)[keys]
    vv = _f64(v)[keys]
    do = _f64(dout_t)
    sk = np.full(H, -np.inf) if sink is None else _f64(sink).reshape(H)
    if len(keys) == 0:  # empty key set: out = 0, lse = sink, no gradient
        z = np.zeros
        return (z(q_t.shape), z((0, q_t.shape[1])), z((0, vv.shape[1])), z(H), z(H),
                z((H, vv.shape[1])), sk.copy())
    s = scale * (q_t @ kk.T)                               # [H, n]
    m = np.maximum(s.max(axis=1), sk)
    z = np.exp(s - m[:, None]).sum(axis=1) + np.exp(sk - m)
    lse = m + np.log(z)
    p = np.exp(s - lse[:, None])                           # [H, n]
    out = p @ vv                                           # [H, Dv]
    dp = do @ vv.T                                         # [H, n]
    delta = (do * out).sum(axis=1)                         # [H]
    ds = p * (dp - delta[:, None])
    dq_t = scale * (ds @ kk)
    dk_part = scale * (ds.T @ q_t)
    dv_part = p.T @ do
    psink = np.exp(sk - lse)
    dsink_part = -psink * delta
    return dq_t, dk_part, dv_part, dsink_part, delta, out, lse


def _bwd(q, k, v, dout, cu_seqlens, sink, scale, keyfn):
    q = _f64(q)
    T, H, Dk = q.shape
    kf = _f64(k)
    vf = _f64(v)
    Dv = vf.shape[1]
    do = _f64(dout)
    sc = _scale(scale, Dk)
    dq = np.zeros((T, H, Dk))
    dk = np.zeros((kf.shape[0], Dk))
    dv = np.zeros((vf.shape[0], Dv))
    dsink = np.zeros(H)
    delta = np.zeros((T, H))
    for bos, eos in doc_bounds(cu_seqlens):
        for t in range(bos, eos):
            keys = keyfn(t, bos, eos)
            dq[t], dkp, dvp, dsp, delta[t], _, _ = attend_bwd(q[t], keys, kf, vf, sink, sc, do[t])
            dk[keys] += dkp
            dv[keys] += dvp
            dsink += dsp
    return {"dq": dq, "dk": dk, "dv": dv, "dsink": dsink if sink is not None else None,
            "delta": delta}


def sparse_mqa_bwd(q, k, v, dout, idx, cu_seqlens, block_size: int, sink=None,
                   scale=None):
    """Backward of the block-sparse MQA forward ([HS] "Core": block-sparse
    DSA gather with an analytic attn_sink gradient).  ``idx`` [T, K] is the
    same per-query block list the forward used.  Returns dict(dq [T,H,Dk],
    dk [T,Dk], dv [T,Dv], dsink [H] or None without a sink, delta [T,H])."""
    idx = np.asarray(idx)

    def keys(t, bos, eos):
        return sparse_key_set(t, bos, eos, idx[t], block_size)

    return _bwd(q, k, v, dout, cu_seqlens, sink, scale, keys)


def swa_mqa_bwd(q, k, v, dout, cu_seqlens, window: int, sink=None, scale=None):
    """Backward of the sliding-window MQA forward ([HS] per-file table:
    windowed MQA fwd/bwd with Dk != Dv and attn_sink)."""

    def keys(t, bos, eos):
        return window_key_set(t, bos, window)

    return _bwd(q, k, v, dout, cu_seqlens, sink, scale, keys)


def dense_causal_bwd(q, k, v, dout, cu_seqlens, sink=None, scale=None):
    """Backward of dense causal MQA with sink inside each document: the
    reference point for full-coverage sparse and wide-window SWA."""

    def keys(t, bos, eos):
        return np.arange(bos, t + 1, dtype=np.int64)

    return _bwd(q, k, v, dout, cu_seqlens, sink, scale, keys)
