"""Independent fp64 restatements used to pin the oracle (test-side only).

Nothing here is imported by the oracle or by the CUDA path, and nothing here
imports either of them.  Each function computes a quantity the oracle must
reproduce, by a different route:

* ``scan_permutation``: the four scan orders as numpy flips/transposes of the
  index grid (GTR news article, section "单向扫描的致命缺陷，以及GTR怎么补").
* ``brute_force``: the O(N^2) closed form of the key-decay recurrence,
      o_t = sum_{s<=t} sum_i q_ti (prod_{r=s+1..t} a_ri) k_si v_s
            + sum_i q_ti (prod_{r=0..t} a_ri) S0[i,:],
  with a_t = exp(g_t) decaying key channels only (same article, section
  "线性注意力到底在省什么").
* ``linear_attention_prefix``: the a == 1 special case, causal linear attention
  by prefix sums.
* ``chunkwise``: the chunked form of the same recurrence (same article,
  section "速度到底快在哪，TensorRT部署做了什么": parallel work inside a chunk,
  only the boundary state carried from chunk to chunk), written with 16-token
  sub-blocks and decay factors that never exceed 1 off the diagonal sub-blocks.
* ``chunkwise_backward``: the gradients of <dO, o> + <dS_f, S_final> in chunked form
  (chunk states by a forward scan, state gradients by a reverse scan, per-chunk
  products, and dg from the suffix sums of q*dq - k*dk), the running log-decay kept
  as (count of zero gates, sum of the other log-decays) and channels whose chunk
  decay is very strong taking one exponential per pair -- the algebra of the
  backward kernels, set against the oracle's position-by-position backward.
"""
from __future__ import annotations

import numpy as np


def scan_permutation(H: int, W: int, direction: int) -> np.ndarray:
    """perm[p] = memory token index visited at scan position p."""
    idx = np.arange(H * W).reshape(H, W)
    if direction == 0:      # L->R, row-major
        grid = idx
    elif direction == 1:    # R->L: rows top to bottom, each row right to left
        grid = idx[:, ::-1]
    elif direction == 2:    # T->B: columns left to right, each column top to bottom
        grid = idx.T
    elif direction == 3:    # B->T: columns left to right, each column bottom to top
        grid = idx[::-1, :].T
    else:
        raise ValueError(direction)
    return np.ascontiguousarray(grid).reshape(-1)


def _sequences(x, perm):
    """[B, N, heads, d] -> list over (b, h) of scan-ordered [N, d] arrays."""
    B, N, heads, d = x.shape
    return [x[b, perm, h, :] for b in range(B) for h in range(heads)]


def brute_force(q, k, v, g, H, W, direction, s0=None):
    """O(N^2 dk) closed form; returns (out [B,N,heads,dv], s_final [B,heads,dk,dv])."""
    q, k, v, g = (np.asarray(t, dtype=np.float64) for t in (q, k, v, g))
    B, N, heads, dk = q.shape
    dv = v.shape[-1]
    perm = scan_permutation(H, W, direction)
    out = np.zeros((B, N, heads, dv))
    sf = np.zeros((B, heads, dk, dv))
    for b in range(B):
        for h in range(heads):
            Q, K, V, A = q[b, perm, h], k[b, perm, h], v[b, perm, h], np.exp(g[b, perm, h])
            S0 = np.zeros((dk, dv)) if s0 is None else np.asarray(s0[b, h], np.float64)
            for t in range(N):
                w = np.ones(dk)          # prod_{r=s+1..t} a_r, built from s = t down
                acc = np.zeros(dv)
                for s in range(t, -1, -1):
                    acc += np.dot(Q[t] * w, K[s]) * V[s]
                    w = w * A[s]
                acc += (Q[t] * w) @ S0   # w = prod_{r=0..t} a_r
                out[b, perm[t], h] = acc
            w = np.ones(dk)
            S = np.zeros((dk, dv))
            for s in range(N - 1, -1, -1):
                S += np.outer(w * K[s], V[s])
                w = w * A[s]
            sf[b, h] = S + w[:, None] * S0
    return out, sf


def linear_attention_prefix(q, k, v, H, W, direction, s0=None):
    """a == 1: o_t = q_t (S0 + sum_{s<=t} k_s^T v_s), by a cumulative sum."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, N, heads, dk = q.shape
    dv = v.shape[-1]
    perm = scan_permutation(H, W, direction)
    out = np.zeros((B, N, heads, dv))
    sf = np.zeros((B, heads, dk, dv))
    for b in range(B):
        for h in range(heads):
            Q, K, V = q[b, perm, h], k[b, perm, h], v[b, perm, h]
            S0 = np.zeros((dk, dv)) if s0 is None else np.asarray(s0[b, h], np.float64)
            states = np.cumsum(K[:, :, None] * V[:, None, :], axis=0) + S0[None]
            out[b, perm, h] = np.einsum("ti,tij->tj", Q, states)
            sf[b, h] = states[-1]
    return out, sf


def chunkwise(q, k, v, g, H, W, direction, s0=None, chunk=64, sub=16):
    """Chunked fp64 restatement; must equal the token-by-token recurrence.

    Per chunk of ``chunk`` scan positions (the tail is padded with q=k=v=0,
    g=0), split into sub-blocks of ``sub`` tokens, with a = exp(g):
      pi[t]  = prod of a over the sub-block from its first token to t (inclusive)
      sig[s] = prod of a over the sub-block strictly after s
      T[L]   = prod of a over sub-block L
    inter-chunk : O += (Q * pi * prod_{L<I} T[L]) @ S_prev
    intra-chunk : score(t in I, s in J<=I) = sum_i Q_ti K_si sig_si * c_ti,
                  c = pi * prod_{J<L<I} T[L]  (I > J, all factors <= 1)
                  c = pi / T[J]               (I == J, the diagonal sub-block)
                  masked to s <= t, then O += scores @ V
    state       : S = prod_L T[L] * S_prev + (K * sig * prod_{L>J} T[L])^T V
    """
    q, k, v, g = (np.asarray(t, dtype=np.float64) for t in (q, k, v, g))
    B, N, heads, dk = q.shape
    dv = v.shape[-1]
    sub = min(sub, chunk)
    assert chunk % sub == 0
    nb = chunk // sub
    perm = scan_permutation(H, W, direction)
    out = np.zeros((B, N, heads, dv))
    sf = np.zeros((B, heads, dk, dv))
    nchunks = -(-N // chunk)
    for b in range(B):
        for h in range(heads):
            S = np.zeros((dk, dv)) if s0 is None else np.array(s0[b, h], np.float64)
            for c in range(nchunks):
                p0, p1 = c * chunk, min((c + 1) * chunk, N)
                n = p1 - p0
                Q = np.zeros((chunk, dk)); K = np.zeros((chunk, dk))
                V = np.zeros((chunk, dv)); G = np.zeros((chunk, dk))
                rows = perm[p0:p1]
                Q[:n], K[:n], V[:n], G[:n] = (q[b, rows, h], k[b, rows, h],
                                              v[b, rows, h], g[b, rows, h])
                A = np.exp(G)
                blk = A.reshape(nb, sub, dk)
                pi = np.cumprod(blk, axis=1).reshape(chunk, dk)
                rev = np.cumprod(blk[:, ::-1, :], axis=1)[:, ::-1, :]   # inclusive suffix
                sig = np.concatenate([rev[:, 1:, :], np.ones((nb, 1, dk))], axis=1)
                sig = sig.reshape(chunk, dk)
                T = np.prod(blk, axis=1)                                # [nb, dk]
                blk_of = np.arange(chunk) // sub
                before = np.array([np.prod(T[:I], axis=0) for I in range(nb)])
                after = np.array([np.prod(T[I + 1:], axis=0) for I in range(nb)])
                O = (Q * pi * before[blk_of]) @ S
                Ksig = K * sig
                scores = np.zeros((chunk, chunk))
                for J in range(nb):
                    cols = slice(J * sub, (J + 1) * sub)
                    for I in range(J, nb):
                        rws = slice(I * sub, (I + 1) * sub)
                        if I == J:
                            cq = pi[rws] / T[J]
                        else:
                            cq = pi[rws] * np.prod(T[J + 1:I], axis=0)
                        scores[rws, cols] = (Q[rws] * cq) @ Ksig[cols].T
                scores = np.tril(scores)
                O += scores @ V
                out[b, rows, h] = O[:n]
                S = np.prod(T, axis=0)[:, None] * S + (Ksig * after[blk_of]).T @ V
            sf[b, h] = S
    return out, sf


def chunkwise_backward(q, k, v, g, dout, H, W, direction, s0=None, dsf=None, chunk=64, fast_range=60.0,
                       zero_gate=-80.0):
    """Chunked fp64 restatement of the backward; returns (dq, dk, dv, dg, ds0).

    Per chunk c (h_c the state entering the chunk, dh_{c+1} the gradient of the state
    leaving it; the running sum b of g from the chunk start kept as the count K of zero
    gates, g <= zero_gate, and the sum R of the other g's; e(t, s) = e^{b_t - b_s} =
    exp(R_t - R_s) if K_t == K_s else 0; B the chunk's total):
      h_{c+1} = e^B h_c + sum_s (k_s e^{B-b_s})^T v_s;   dh_c = e^B dh_{c+1} + sum_t (q_t e^{b_t})^T dO_t
      D[t,s] = dO_t . v_s,  A[t,s] = sum_i q_ti k_si e(t, s)_i   (s <= t)
      dq_t = e^{b_t} (dO_t h_c^T) + sum_{s<=t} D[t,s] k_s e(t, s)
      dk_s = e^{B-b_s} (v_s dh_{c+1}^T) + sum_{t>=s} D[t,s] q_t e(t, s)
      dv_s = sum_{t>=s} A[t,s] dO_t + (k_s e^{B-b_s}) dh_{c+1}
      dg_r = sum_{t>=r} (q_t dq_t - k_t dk_t) + sum_j dS_f[:, j] S_final[:, j]
    The intra-chunk factors use e^{R_t} e^{-R_s} for channels with no zero gate in the
    chunk and R_63 >= -fast_range, and e(t, s) directly for the others.
    """
    q, k, v, g, dout = (np.asarray(t, dtype=np.float64) for t in (q, k, v, g, dout))
    B_, N, heads, dk = q.shape
    dv = v.shape[-1]
    perm = scan_permutation(H, W, direction)
    nc = -(-N // chunk)
    dq, dkk, dg = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    dvv = np.zeros_like(v)
    ds0 = np.zeros((B_, heads, dk, dv))
    mask = np.tril(np.ones((chunk, chunk)))

    def e_ts(t):    # [chunk, chunk, dk]: e(t, s) for s <= t, 0 above the diagonal
        same = t["K"][:, None, :] == t["K"][None, :, :]
        diff = np.minimum(t["R"][:, None, :] - t["R"][None, :, :], 0.0)
        return np.where(same, np.exp(diff), 0.0) * mask[:, :, None]

    for b in range(B_):
        for h in range(heads):
            tiles = []
            for c in range(nc):
                rows = perm[c * chunk:(c + 1) * chunk]
                n = len(rows)
                t = {}
                for name, x in (("q", q), ("k", k), ("g", g), ("v", v), ("do", dout)):
                    m = np.zeros((chunk, x.shape[-1]))
                    m[:n] = x[b, rows, h]
                    t[name] = m
                zg = t["g"] <= zero_gate
                t["K"] = np.cumsum(zg, axis=0)
                t["R"] = np.cumsum(np.where(zg, 0.0, t["g"]), axis=0)
                t["eB"] = np.where(t["K"][-1] == 0, np.exp(t["R"][-1]), 0.0)             # e^B
                t["eb"] = np.where(t["K"] == 0, np.exp(t["R"]), 0.0)                     # e^{b_t}
                t["eBb"] = np.where(t["K"][-1] == t["K"], np.exp(t["R"][-1] - t["R"]), 0.0)   # e^{B-b_s}
                t["rows"] = rows
                tiles.append(t)
            S0 = np.zeros((dk, dv)) if s0 is None else np.asarray(s0[b, h], np.float64)
            hs, hcur = [], S0
            for t in tiles:   # forward scan of the chunk states
                hs.append(hcur)
                hcur = t["eB"][:, None] * hcur + (t["k"] * t["eBb"]).T @ t["v"]
            SN = hcur
            dS = np.zeros((dk, dv)) if dsf is None else np.asarray(dsf[b, h], np.float64)
            const = (dS * SN).sum(axis=1)
            dhs = [None] * nc
            dcur = dS
            for c in range(nc - 1, -1, -1):   # reverse scan of the state gradients
                t = tiles[c]
                dhs[c] = dcur
                dcur = t["eB"][:, None] * dcur + (t["q"] * t["eb"]).T @ t["do"]
            ds0[b, h] = dcur
            xs = []
            for c, t in enumerate(tiles):
                Q, K, V, DO = t["q"], t["k"], t["v"], t["do"]
                fast = (t["K"][-1] == 0) & (t["R"][-1] >= -fast_range)
                D = (DO @ V.T) * mask
                qh = np.where(fast, Q * np.exp(t["R"]), 0.0)
                with np.errstate(over="ignore", invalid="ignore"):
                    kh = np.where(fast, K * np.exp(-t["R"]), 0.0)
                    y2 = np.where(fast, np.exp(-t["R"]) * (D.T @ qh), 0.0)
                A = (qh @ kh.T) * mask
                dq_c = t["eb"] * (DO @ hs[c].T) + np.where(fast, np.exp(t["R"]), 0.0) * (D @ kh)
                dk_c = t["eBb"] * (V @ dhs[c].T) + y2
                slow = np.where(~fast)[0]
                if len(slow):
                    E = e_ts(t)
                    for i in slow:
                        A += np.outer(Q[:, i], K[:, i]) * E[:, :, i]
                        dq_c[:, i] += (D * E[:, :, i]) @ K[:, i]
                        dk_c[:, i] += (D * E[:, :, i]).T @ Q[:, i]
                dv_c = A.T @ DO + (K * t["eBb"]) @ dhs[c]
                x = Q * dq_c - K * dk_c
                n = len(t["rows"])
                dq[b, t["rows"], h] = dq_c[:n]
                dkk[b, t["rows"], h] = dk_c[:n]
                dvv[b, t["rows"], h] = dv_c[:n]
                xs.append(np.flip(np.cumsum(np.flip(x, 0), 0), 0))
            for c, t in enumerate(tiles):
                off = const + sum(xs[c2][0] for c2 in range(c + 1, nc))
                dg[b, t["rows"], h] = (xs[c] + off)[:len(t["rows"])]
    return dq, dkk, dvv, dg, ds0
