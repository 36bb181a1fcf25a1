"""One layer of the decode step restated in numpy with the mirror mode's roundings.

Used only to pin the oracle's mirror mode (tests/test_oracle.py): it writes the layer
equations out again from their definitions, with bf16 round-to-nearest-even applied at each
storage point of the GPU path, and shares no code with the oracle beyond the dequantized
weight matrices (pinned on their own by the code round-trip tests).  Storage points:

  P1  u = bf16(r * gamma), with the row's 1/rms applied to the dot products
  P2  in_proj output z | xBC | dt_raw rounded to bf16
  P4  gated-norm output bf16(v * gamma_n), with the group's 1/rms applied to the dot products
  P5  q, k, v rounded to bf16
  P6  attention output rounded to bf16
  P7  squared-ReLU hidden rounded to bf16
  P8  final norm as P1 with gamma_f
The residual stream and the SSM state stay unrounded.
"""
import numpy as np

import synth


def bf16(v):
    """round float64 values to the nearest bf16 value, ties to even (8 significant bits)"""
    v = np.asarray(v, np.float64)
    m, e = np.frexp(v)                 # v = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)


def silu(x):
    return x / (1.0 + np.exp(-x))


def softplus(x):
    return np.logaddexp(0.0, x)


def _norm_in(r, gamma, eps):
    """P1: (bf16(r * gamma), 1/rms of r) for each row of r [B][d]"""
    inv = 1.0 / np.sqrt(np.mean(r * r, axis=-1, keepdims=True) + eps)
    return bf16(r * gamma[None, :]), inv


def layer(model, state, l, r_in, slots):
    """Layer l of the step on the residual rows r_in [B][d] (float64); state is an oracle.State
    (double arrays) that is updated in place like the oracle does.  Returns the residual leaving
    the layer."""
    cfg = model.cfg
    sp = model.small[l]
    eps = cfg.eps
    kind = cfg.pattern[l]
    mi = cfg.pattern[:l].count("M")
    ai = cfg.pattern[:l].count("*")
    r = np.array(r_in, np.float64)
    un, inv = _norm_in(r, sp["norm"].astype(np.float64), eps)
    if kind == "M":
        H, P, N, G, W = cfg.ssm_heads, cfg.ssm_head_dim, cfg.ssm_state, cfg.ssm_groups, cfg.conv_width
        E, Cx, NG = cfg.d_inner, cfg.conv_dim, cfg.norm_groups
        Win = model.mats[(l, synth.K_IN)].dequant()
        Wout = model.mats[(l, synth.K_OUT)].dequant()
        zx = bf16((un @ Win.T) * inv)                                  # P2
        cw = sp["conv_w"].astype(np.float64)                           # [Cx][W], column W-1 newest
        A = -np.exp(sp["A_log"].astype(np.float64))
        Ulist = []
        for b, s in enumerate(slots):
            z, xBC, dtr = zx[b, :E], zx[b, E:E + Cx], zx[b, E + Cx:]
            hist = state.conv[mi, s]                                   # [W-1][Cx], oldest first
            window = np.vstack([hist, xBC[None, :]])                   # [W][Cx]
            xc = silu(sp["conv_b"].astype(np.float64) + np.sum(cw.T * window, axis=0))
            state.conv[mi, s] = window[1:]
            x, Bv, Cv = xc[:E].reshape(H, P), xc[E:E + G * N].reshape(G, N), xc[E + G * N:].reshape(G, N)
            dt = softplus(dtr + sp["dt_bias"].astype(np.float64))
            S = state.ssm[mi, s]                                       # [H][P][N]
            y = np.empty((H, P))
            for h in range(H):
                g = h * G // H
                S[h] = np.exp(A[h] * dt[h]) * S[h] + dt[h] * np.outer(x[h], Bv[g])
                y[h] = S[h] @ Cv[g] + sp["D"][h] * x[h]
            v = y.reshape(E) * silu(z)
            gs = E // NG
            u = np.empty(E)
            for q in range(NG):
                c = slice(q * gs, (q + 1) * gs)
                iq = 1.0 / np.sqrt(np.mean(v[c] * v[c]) + eps)
                u[c] = bf16(v[c] * sp["gnorm"][c].astype(np.float64)) * iq   # P4
            Ulist.append(u)
        return r + np.stack(Ulist) @ Wout.T
    if kind == "*":
        Hq, Hk, Dh = cfg.attn_q_heads, cfg.attn_kv_heads, cfg.attn_head_dim
        Wqkv = model.mats[(l, synth.K_QKV)].dequant()
        Wo = model.mats[(l, synth.K_O)].dequant()
        qkv = bf16((un @ Wqkv.T) * inv)                                # P5
        O = []
        for b, s in enumerate(slots):
            t = int(state.ctx_len[s])
            q = qkv[b, :Hq * Dh].reshape(Hq, Dh)
            state.k[ai, s, :, t] = qkv[b, Hq * Dh:(Hq + Hk) * Dh].reshape(Hk, Dh)
            state.v[ai, s, :, t] = qkv[b, (Hq + Hk) * Dh:].reshape(Hk, Dh)
            o = np.empty((Hq, Dh))
            for i in range(Hq):
                j = i * Hk // Hq
                sc = state.k[ai, s, j, :t + 1] @ q[i] / np.sqrt(Dh)
                p = np.exp(sc - sc.max())
                o[i] = bf16((p / p.sum()) @ state.v[ai, s, j, :t + 1])    # P6
            O.append(o.reshape(Hq * Dh))
        return r + np.stack(O) @ Wo.T
    Wup = model.mats[(l, synth.K_UP)].dequant()
    Wdn = model.mats[(l, synth.K_DOWN)].dequant()
    h = bf16(np.maximum((un @ Wup.T) * inv, 0.0) ** 2)                 # P7
    return r + h @ Wdn.T


def heads(model, r):
    """P8 and both heads: (logits_text [B][Vt], logits_func [B][Vf])"""
    un, inv = _norm_in(np.asarray(r, np.float64), model.final_norm.astype(np.float64), model.cfg.eps)
    return (un @ model.head_text.dequant().T) * inv, (un @ model.head_func.dequant().T) * inv
