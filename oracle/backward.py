"""Gradients of sink-augmented GQA attention, written out in fp64.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

GPT-OSS-Lite README: the sinks are learned attention parameters and the
model trains end to end ("Architecture": learned attention sinks; the
training pipeline), so the attention needs its backward pass. The pages give
no gradient formulas; these are the derivatives of the forward the oracle
defines (``attention.sink_attention``), for one call with no cache prefix
(offset 0: a training sequence attends to itself), on the rotated q and k:

    s_ij   = sm_scale <q_i, k_j>            (admitted pairs; others -inf)
    L_i    = sum_j e^{s_ij} + e^{sigma}     lse_i = ln L_i
    P_ij   = e^{s_ij} / L_i                 P_sink,i = e^{sigma} / L_i
    o_i    = sum_j P_ij v_j                 (the sink column carries no value)

With dO the gradient of the loss with respect to o, and D_i = <dO_i, o_i>:

    dP_ij  = <dO_i, v_j>
    dS_ij  = P_ij (dP_ij - D_i)             (the sink's dP is 0: no value)
    dq_i   = sm_scale sum_j dS_ij k_j
    dk_j   = sm_scale sum_{i, heads of the group} dS_ij q_i
    dv_j   = sum_{i, heads of the group} P_ij dO_i
    dsigma = - sum_{b, i} P_sink,i D_i     (per query head)

GQA sums the contributions of the q_mult query heads that share a KV head.
Gradients with respect to the unrotated q, k are the rotation's transpose
applied to these (a rotation by -theta).
"""

import numpy as np

from .attention import allowed_mask


def attention_backward(q_rot, k_rot, v, sinks, window, sm_scale, d_out):
    """Returns (dq [B,T,n_q,d], dk [B,T,n_kv,d], dv [B,T,n_kv,d], dsinks [n_q]),
    all fp64, for queries and keys at positions 0..T-1 (offset 0)."""
    q_rot = np.asarray(q_rot, dtype=np.float64)
    k_rot = np.asarray(k_rot, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    d_out = np.asarray(d_out, dtype=np.float64)
    B, T, n_q, d = q_rot.shape
    n_kv = k_rot.shape[2]
    q_mult = n_q // n_kv
    sig = np.full(n_q, -np.inf) if sinks is None else np.asarray(sinks, dtype=np.float64)
    ok = allowed_mask(0, T, T, window)
    dq = np.zeros_like(q_rot)
    dk = np.zeros_like(k_rot)
    dv = np.zeros_like(v)
    dsinks = np.zeros(n_q)
    for b in range(B):
        for h in range(n_q):
            g = h // q_mult
            K, V = k_rot[b, :, g, :], v[b, :, g, :]
            s = np.where(ok, (q_rot[b, :, h, :] @ K.T) * sm_scale, -np.inf)
            m = np.maximum(s.max(axis=1), sig[h])
            e = np.exp(s - m[:, None])
            L = e.sum(axis=1) + np.exp(sig[h] - m)
            P = e / L[:, None]
            p_sink = np.exp(sig[h] - m) / L
            o = P @ V
            dO = d_out[b, :, h, :]
            Dv = np.sum(dO * o, axis=1)
            dP = dO @ V.T
            dS = P * (dP - Dv[:, None])
            dq[b, :, h, :] = sm_scale * (dS @ K)
            dk[b, :, g, :] += sm_scale * (dS.T @ q_rot[b, :, h, :])
            dv[b, :, g, :] += P.T @ dO
            dsinks[h] += -np.sum(p_sink * Dv)
    return dq, dk, dv, dsinks
