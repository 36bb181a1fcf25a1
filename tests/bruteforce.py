"""Direct full-sequence evaluation of the hybrid stack in numpy (float64, no rounding).

Used only to pin the oracle: it evaluates every frame of a sequence at once from
the closed forms instead of the per-frame recurrence the oracle steps through:

  * causal depthwise conv1d as a sum over the zero-padded input sequence,
  * the Mamba-2 SSM as its semiseparable matrix (Dao & Gu, "Transformers are
    SSMs", the SSM-as-matrix view):
        y_t = sum_{s<=t} (C_t . B_s) exp(A sum_{r=s+1..t} dt_r) dt_s x_s + D x_t
    for a zero initial state,
  * attention as one masked softmax over the whole sequence,
  * norms, gates and the MLP elementwise over all frames.

Weights are the oracle's dequantized matrices (the dequantization itself is
pinned separately by the code round-trip and constructed-weight tests).
"""
import numpy as np


def silu(x):
    return x / (1.0 + np.exp(-x))


def softplus(x):
    return np.logaddexp(0.0, x)


def rmsnorm(X, gamma, eps):
    return X * gamma / np.sqrt(np.mean(X * X, axis=-1, keepdims=True) + eps)


def full_sequence(model, X):
    """X: [T][d] float64 frame inputs. Returns hidden [L+1][T][d] and logits (text, func) [T][V]."""
    cfg = model.cfg
    T, d = X.shape
    eps = cfg.eps
    H, P, N, G, W = cfg.ssm_heads, cfg.ssm_head_dim, cfg.ssm_state, cfg.ssm_groups, cfg.conv_width
    E, Cx = cfg.d_inner, cfg.conv_dim
    Hq, Hk, Dh = cfg.attn_q_heads, cfg.attn_kv_heads, cfg.attn_head_dim
    import synth

    R = X.astype(np.float64).copy()
    hidden = [R.copy()]
    causal = np.tril(np.ones((T, T), bool))
    for l, kind in enumerate(cfg.pattern):
        sp = model.small[l]
        U = rmsnorm(R, sp["norm"].astype(np.float64), eps)
        if kind == "M":
            Win = model.mats[(l, synth.K_IN)].dequant()
            Wout = model.mats[(l, synth.K_OUT)].dequant()
            Z = U @ Win.T
            z, xBC, dtr = Z[:, :E], Z[:, E:E + Cx], Z[:, E + Cx:]
            cw = sp["conv_w"].astype(np.float64)           # [Cx][W], column W-1 = newest
            padded = np.vstack([np.zeros((W - 1, Cx)), xBC])
            pre = np.tile(sp["conv_b"].astype(np.float64), (T, 1))
            for k in range(W):
                pre += cw[:, k][None, :] * padded[k:k + T]
            xc = silu(pre)
            x, Bm, Cm = xc[:, :E], xc[:, E:E + G * N], xc[:, E + G * N:]
            dt = softplus(dtr + sp["dt_bias"].astype(np.float64)[None, :])   # [T][H]
            A = -np.exp(sp["A_log"].astype(np.float64))
            Y = np.zeros((T, E))
            for h in range(H):
                g = h * G // H
                Bg, Cg = Bm[:, g * N:(g + 1) * N], Cm[:, g * N:(g + 1) * N]
                seg = np.cumsum(A[h] * dt[:, h])                           # sum_{r<=t}
                decay = np.exp(seg[:, None] - seg[None, :])                 # sum_{r=s+1..t}
                Mh = (Cg @ Bg.T) * decay * dt[None, :, h]
                Mh = np.where(causal, Mh, 0.0)
                xh = x[:, h * P:(h + 1) * P]
                Y[:, h * P:(h + 1) * P] = Mh @ xh + sp["D"][h] * xh
            V = Y * silu(z)
            gs = E // cfg.norm_groups
            Vn = np.empty_like(V)
            for q in range(cfg.norm_groups):
                sl = slice(q * gs, (q + 1) * gs)
                Vn[:, sl] = rmsnorm(V[:, sl], sp["gnorm"][sl].astype(np.float64), eps)
            R = R + Vn @ Wout.T
        elif kind == "*":
            Wqkv = model.mats[(l, synth.K_QKV)].dequant()
            Wo = model.mats[(l, synth.K_O)].dequant()
            QKV = U @ Wqkv.T
            Q = QKV[:, :Hq * Dh].reshape(T, Hq, Dh)
            K = QKV[:, Hq * Dh:(Hq + Hk) * Dh].reshape(T, Hk, Dh)
            Vv = QKV[:, (Hq + Hk) * Dh:].reshape(T, Hk, Dh)
            O = np.zeros((T, Hq, Dh))
            for i in range(Hq):
                j = i * Hk // Hq
                S = (Q[:, i, :] @ K[:, j, :].T) / np.sqrt(Dh)
                S = np.where(causal, S, -np.inf)
                S = S - S.max(axis=1, keepdims=True)
                Pm = np.exp(S)
                Pm /= Pm.sum(axis=1, keepdims=True)
                O[:, i, :] = Pm @ Vv[:, j, :]
            R = R + O.reshape(T, Hq * Dh) @ Wo.T
        else:
            Wup = model.mats[(l, synth.K_UP)].dequant()
            Wdn = model.mats[(l, synth.K_DOWN)].dequant()
            Hm = np.maximum(U @ Wup.T, 0.0) ** 2
            R = R + Hm @ Wdn.T
        hidden.append(R.copy())
    Uf = rmsnorm(R, model.final_norm.astype(np.float64), eps)
    lt = Uf @ model.head_text.dequant().T
    lf = Uf @ model.head_func.dequant().T
    return np.stack(hidden), lt, lf
