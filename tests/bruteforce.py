"""Second, independent restatement of the draft forward and verify for tiny inputs.

Pure Python: nested loops over rows, heads and features with ``math`` only.
It exists to pin the NumPy oracle; it is written from the same readings but
shares no code with it (no matmul, no vectorised softmax, explicit indices).
"""

import math


def _row(mat, i):
    return [float(v) for v in mat[i]]


def matvec_out_in(W, x):
    """y[o] = sum_i W[o][i] * x[i] with W stored [out][in]."""
    out = []
    for o in range(len(W)):
        s = 0.0
        Wo = W[o]
        for i in range(len(x)):
            s += float(Wo[i]) * x[i]
        out.append(s)
    return out


def rmsnorm(x, g, eps):
    ms = 0.0
    for v in x:
        ms += v * v
    ms /= len(x)
    inv = 1.0 / math.sqrt(ms + eps)
    return [x[i] * inv * float(g[i]) for i in range(len(x))]


def rope_vec(v, p, base):
    hd = len(v)
    h = hd // 2
    out = [0.0] * hd
    for i in range(h):
        th = base ** (-2.0 * i / hd)
        c, s = math.cos(p * th), math.sin(p * th)
        out[i] = v[i] * c - v[i + h] * s
        out[i + h] = v[i + h] * c + v[i] * s
    return out


def features(tap_rows, W_fc, g_ctx, eps):
    x = []
    for t in tap_rows:
        x.extend(float(v) for v in t)
    return rmsnorm(matvec_out_in(W_fc, x), g_ctx, eps)


def inject_row(c, p, Wk, Wv, nkv, hd, base):
    k = matvec_out_in(Wk, c)
    v = matvec_out_in(Wv, c)
    K = [rope_vec(k[j * hd:(j + 1) * hd], p, base) for j in range(nkv)]
    Vv = [v[j * hd:(j + 1) * hd] for j in range(nkv)]
    return K, Vv


def layer(xs, T, Kc, Vc, lw, cfg):
    """xs: list of B rows; Kc/Vc: [T][nkv][hd] nested lists."""
    B = len(xs)
    nq, nkv, hd, eps, base = cfg.nq, cfg.nkv, cfg.hd, cfg.eps, cfg.rope_base
    grp = nq // nkv
    hs = [rmsnorm(x, lw["g_in"], eps) for x in xs]
    qs, ks, vs = [], [], []
    for j, h in enumerate(hs):
        q = matvec_out_in(lw["Wq"], h)
        k = matvec_out_in(lw["Wk"], h)
        v = matvec_out_in(lw["Wv"], h)
        qs.append([rope_vec(q[a * hd:(a + 1) * hd], T + j, base) for a in range(nq)])
        ks.append([rope_vec(k[a * hd:(a + 1) * hd], T + j, base) for a in range(nkv)])
        vs.append([v[a * hd:(a + 1) * hd] for a in range(nkv)])
    new = []
    for j in range(B):
        o = []
        for a in range(nq):
            kv = a // grp
            keys = [Kc[t][kv] for t in range(T)] + [ks[u][kv] for u in range(B)]
            vals = [Vc[t][kv] for t in range(T)] + [vs[u][kv] for u in range(B)]
            sc = []
            for key in keys:
                s = 0.0
                for e in range(hd):
                    s += qs[j][a][e] * key[e]
                sc.append(s / math.sqrt(hd))
            m = max(sc)
            w = [math.exp(s - m) for s in sc]
            tot = sum(w)
            for e in range(hd):
                acc = 0.0
                for t in range(len(vals)):
                    acc += w[t] * vals[t][e]
                o.append(acc / tot)
        att = matvec_out_in(lw["Wo"], o)
        x = [xs[j][i] + att[i] for i in range(len(att))]
        h2 = rmsnorm(x, lw["g_post"], eps)
        gg = matvec_out_in(lw["Wg"], h2)
        uu = matvec_out_in(lw["Wu"], h2)
        act = [gg[i] / (1.0 + math.exp(-gg[i])) * uu[i] for i in range(len(gg))]
        dn = matvec_out_in(lw["Wd"], act)
        new.append([x[i] + dn[i] for i in range(len(x))])
    return new


def forward_logits(tokens, T, caches, w, cfg):
    """Logits [B][V] of a block (every position), brute force."""
    xs = [_row(w["emb"], int(t)) for t in tokens]
    for l in range(cfg.L):
        Kc, Vc = caches[l]
        xs = layer(xs, T, Kc, Vc, w["layers"][l], cfg)
    zs = [rmsnorm(x, w["g_final"], cfg.eps) for x in xs]
    return [matvec_out_in(w["W_lm"], z) for z in zs]


def argmax_first(row):
    best, bi = None, -1
    for i, v in enumerate(row):
        if best is None or v > best:
            best, bi = v, i
    return bi


def accept_all_prefixes(g, draft):
    """Accept length by trying every prefix length from longest to shortest."""
    B = len(draft)
    for a in range(B - 1, -1, -1):
        if all(int(g[i]) == int(draft[i + 1]) for i in range(a)):
            return a
    return 0
