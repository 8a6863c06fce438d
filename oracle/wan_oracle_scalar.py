"""Scalar-loop fp64 oracle of one WanAttentionBlock and the CFG-Euler step,
for the tiny configuration: plain Python floats and the ``math`` module, no
arrays and no BLAS, one token row and one multiply-add at a time, in the
order the pages give the steps, so that it can be checked against them by
eye.

TEST INFRASTRUCTURE ONLY, like ``oracle.wan_oracle``: only the tests import
it. It shares no code with the CUDA library nor with ``oracle.wan_oracle``
(its own RoPE frequencies, norms, attention and GELU). It is slow (pure
Python): sized for grids of a few dozen tokens.

Sources:
* "Wan2.2 code walkthrough" (newtid.com): WanAttentionBlock core-logic
  snippet (modulation chunks, the three branches and their residuals), 3D
  RoPE snippet (pairs split [c - 2(c//3), c//3, c//3] between t, h, w,
  interleaved real / imaginary parts), self-attention snippet (softmax over
  every key, no causal mask), structure snippet (qk_norm, cross_attn_norm,
  GELU tanh), sampling-loop snippet (classifier-free guidance).
* "Wan paper deep dive" (charles2530.github.io), "Video DiT and Flow
  Matching": the Euler move along the velocity.

Readings where the pages are silent are the same as ``oracle.wan_oracle``'s:
per-axis frequency ladders theta^(-2j/d_a), 0-based grid positions, RMSNorm
of q and k over the full model width, population variance with eps inside
the root, softmax scale 1/sqrt(d), a bias on every linear layer, a row with
no valid key gives zeros.

Data layout: a matrix is a list of rows (lists of floats); weights are
[out][in] like ``nn.Linear``; a sequence is a list of token rows.
"""
from __future__ import annotations

import math


def _tolist(a):
    """Nested Python lists of floats (accepts numpy arrays or lists)."""
    if hasattr(a, "tolist"):
        a = a.tolist()
    return a


def linear_row(a, w, b):
    """y_o = sum_i a_i W[o][i] + b_o, one output at a time."""
    out = []
    for o in range(len(w)):
        acc = 0.0
        row = w[o]
        for i in range(len(a)):
            acc += a[i] * row[i]
        out.append(acc + (b[o] if b is not None else 0.0))
    return out


def layer_norm_row(x, eps, gamma=None, beta=None):
    n = len(x)
    mean = 0.0
    for v in x:
        mean += v
    mean /= n
    var = 0.0
    for v in x:
        var += (v - mean) * (v - mean)
    var /= n
    inv = 1.0 / math.sqrt(var + eps)
    out = []
    for i in range(n):
        y = (x[i] - mean) * inv
        if gamma is not None:
            y *= gamma[i]
        if beta is not None:
            y += beta[i]
        out.append(y)
    return out


def rms_norm_row(x, gamma, eps):
    ss = 0.0
    for v in x:
        ss += v * v
    inv = 1.0 / math.sqrt(ss / len(x) + eps)
    return [x[i] * inv * gamma[i] for i in range(len(x))]


def gelu_tanh(z):
    return 0.5 * z * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z * z * z)))


def rope_rotate_head(v, t, h, w, theta):
    """Rotate one head vector (length d) of the token at grid (t, h, w): pair
    j = (v[2j], v[2j+1]) turns by pos * theta^(-2 j' / d_a), where the pair
    belongs to the t axis for its first c - 2(c//3) pairs, then h, then w,
    j' is its index within the axis and d_a twice the axis's pair count."""
    d = len(v)
    c = d // 2
    counts = (c - 2 * (c // 3), c // 3, c // 3)
    positions = (t, h, w)
    out = list(v)
    j = 0
    for axis in range(3):
        p = counts[axis]
        for jj in range(p):
            ang = positions[axis] * theta ** (-(2.0 * jj) / (2 * p))
            cs, sn = math.cos(ang), math.sin(ang)
            re, im = v[2 * j], v[2 * j + 1]
            out[2 * j] = re * cs - im * sn
            out[2 * j + 1] = re * sn + im * cs
            j += 1
    return out


def attention_row(q_heads, k_rows, v_rows, k_len, scale):
    """One query token: for each head, softmax over the first k_len keys of
    q . k_j * scale, then the weighted sum of the values. q_heads [n][d],
    k_rows / v_rows [Lk][n][d]."""
    n = len(q_heads)
    d = len(q_heads[0])
    out = []
    for hh in range(n):
        if k_len == 0:
            out.append([0.0] * d)
            continue
        s = []
        for j in range(k_len):
            acc = 0.0
            for e in range(d):
                acc += q_heads[hh][e] * k_rows[j][hh][e]
            s.append(acc * scale)
        m = max(s)
        p = [math.exp(sj - m) for sj in s]
        tot = 0.0
        for pj in p:
            tot += pj
        o = [0.0] * d
        for j in range(k_len):
            wj = p[j] / tot
            for e in range(d):
                o[e] += wj * v_rows[j][hh][e]
        out.append(o)
    return out


def _heads(vec, n):
    d = len(vec) // n
    return [vec[hh * d:(hh + 1) * d] for hh in range(n)]


def _flat(heads):
    return [v for head in heads for v in head]


def block_forward(x, ctx, ctx_len, e0, w, heads, grid, eps, theta=1e4):
    """One block on one sequence: x [L][D], ctx [T][D], e0 [6][D] (one
    timestep for the sequence), weights by the names of ``wan_block_weights``.
    Returns the new x [L][D]."""
    x = [list(r) for r in _tolist(x)]
    ctx = _tolist(ctx)
    e0 = _tolist(e0)
    w = {k: _tolist(v) for k, v in w.items()}
    F, H, W = grid
    L, D = len(x), len(x[0])
    T = len(ctx)
    d = D // heads
    scale = 1.0 / math.sqrt(d)
    klen = T if ctx_len is None else int(ctx_len)
    # modulation chunks: m_k = modulation[k] + e0[k]
    m = [[w["modulation"][k][i] + e0[k][i] for i in range(D)] for k in range(6)]

    # ---- self-attention: every token's q, k, v first (keys need all rows)
    qs, ks, vs = [], [], []
    for i in range(L):
        t, hh, ww = i // (H * W), (i // W) % H, i % W
        u = layer_norm_row(x[i], eps)
        u = [u[c] * (1.0 + m[1][c]) + m[0][c] for c in range(D)]
        q = rms_norm_row(linear_row(u, w["wq"], w["bq"]), w["gq"], eps)
        k = rms_norm_row(linear_row(u, w["wk"], w["bk"]), w["gk"], eps)
        v = linear_row(u, w["wv"], w["bv"])
        qs.append([rope_rotate_head(hd, t, hh, ww, theta) for hd in _heads(q, heads)])
        ks.append([rope_rotate_head(hd, t, hh, ww, theta) for hd in _heads(k, heads)])
        vs.append(_heads(v, heads))
    for i in range(L):
        o = _flat(attention_row(qs[i], ks, vs, L, scale))
        y = linear_row(o, w["wo"], w["bo"])
        x[i] = [x[i][c] + m[2][c] * y[c] for c in range(D)]

    # ---- cross-attention (ungated), keys and values from the context
    kc, vc = [], []
    for j in range(T):
        kc.append(_heads(rms_norm_row(linear_row(ctx[j], w["cwk"], w["cbk"]), w["cgk"], eps), heads))
        vc.append(_heads(linear_row(ctx[j], w["cwv"], w["cbv"]), heads))
    for i in range(L):
        a3 = layer_norm_row(x[i], eps, w["g3"], w["b3"])
        qc = _heads(rms_norm_row(linear_row(a3, w["cwq"], w["cbq"]), w["cgq"], eps), heads)
        oc = _flat(attention_row(qc, kc, vc, klen, scale))
        y = linear_row(oc, w["cwo"], w["cbo"])
        x[i] = [x[i][c] + y[c] for c in range(D)]

    # ---- FFN
    for i in range(L):
        a2 = layer_norm_row(x[i], eps)
        a2 = [a2[c] * (1.0 + m[4][c]) + m[3][c] for c in range(D)]
        hdn = [gelu_tanh(z) for z in linear_row(a2, w["w1"], w["b1"])]
        y = linear_row(hdn, w["w2"], w["b2"])
        x[i] = [x[i][c] + m[5][c] * y[c] for c in range(D)]
    return x


def euler_cfg_step(x, v_cond, v_uncond, guide_scale, sigma, sigma_next):
    """x + (sigma' - sigma) (v_u + s (v_c - v_u)), element by element."""
    dt = sigma_next - sigma
    return [x[i] + dt * (v_uncond[i] + guide_scale * (v_cond[i] - v_uncond[i])) for i in range(len(x))]
