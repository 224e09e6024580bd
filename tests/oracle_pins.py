"""Pins for the CPU oracle: checks against facts that do not come from the oracle.

Each ``pin_*`` takes a loaded oracle library handle and raises AssertionError
when the oracle disagrees with what the pages or the mathematics fix.  The same
functions run against the real oracle (``test_oracle.py``: all must pass) and
against copies of it with a planted mistake (``test_oracle_mutants.py``: at
least one must fail for each mistake).

Sources (page title, section):
* paper summary of arXiv 2603.15619, "Mixture-of-Depths Attention (MoDA): The
  Unified Operator" -- the joint-softmax equation, the grouped causal mask
  floor(i_q/G) >= i_k and the depth matching mask floor(i_q/G) == floor(j_d/L)
  in the flattened query-row index i_q = t*G + g;
* same section, "The depth KV at different layers" -- with no depth history
  MoDA is plain causal self-attention;
* same summary, "Fused online-softmax (Algorithm 1)" -- the base-2 running
  max / sum / output update over G-aligned query blocks, two sequence phases
  then the depth loop, and the statement that online softmax is exact;
* "moda-attention 0.1.0" PyPI page, "Key Design Choices" -- GQA expansion by
  repeat_interleave; "Using the Kernel Directly" -- tensor layouts;
* paper summary, "Hardware-Efficient Implementation" -- token t's L depth rows
  sit at [t*L, (t+1)*L) of the flattened depth tensor;
* ByteDance-Seed/MoDA README, "TODO" (non-causal MoDA kernel) and paper
  summary, "7. Implications and Future Directions" (vision use) -- the
  non-causal operator drops the sequence mask and keeps the depth mask;
* paper summary, "6. Limitations and Trade-offs" (bounded depth-KV slots,
  sliding-window recency) -- a depth window keeps each token's last S layers.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

LOG2E = 1.0 / math.log(2.0)


# ---------------------------------------------------------------- inputs ----
def rand_case(B, Hq, Hk, T, d, L, seed, dtype=torch.float64):
    """Small fp64 inputs (plain N(0,1)); depth already token-major."""
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(B, Hq, T, d, generator=g, dtype=dtype)
    K = torch.randn(B, Hk, T, d, generator=g, dtype=dtype)
    V = torch.randn(B, Hk, T, d, generator=g, dtype=dtype)
    Kd = torch.randn(B, Hk, T * L, d, generator=g, dtype=dtype)
    Vd = torch.randn(B, Hk, T * L, d, generator=g, dtype=dtype)
    dO = torch.randn(B, Hq, T, d, generator=g, dtype=dtype)
    return Q, K, V, Kd, Vd, dO


# ------------------------------------------ independent dense formulation ----
def dense_moda(Q, K, V, Kd, Vd, scale=None, causal=True, window=0):
    """The 'naive' dense form: concatenate [K | K_depth], build the full mask
    matrix M in the flattened row index i_q = t*G + g, one softmax per row.
    causal=False drops the sequence mask; window > 0 keeps depth column j_d
    only if its layer j_d mod L is among the token's last `window` layers.
    Pure torch library ops (differentiable), fp64."""
    B, Hq, T, d = Q.shape
    Hk = K.shape[1]
    G = Hq // Hk
    L = Kd.shape[2] // T if T else 0
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    # rows of one KV head's group, flattened as i_q = t*G + g
    Qf = Q.reshape(B, Hk, G, T, d).permute(0, 1, 3, 2, 4).reshape(B, Hk, T * G, d)
    i_q = torch.arange(T * G)
    t_base = i_q // G
    seq_mask = t_base[:, None] >= torch.arange(T)[None, :]
    if not causal:
        seq_mask = torch.ones_like(seq_mask)
    j_d = torch.arange(T * L)
    dep_mask = t_base[:, None] == (j_d // max(L, 1))[None, :]
    if window:
        dep_mask &= ((j_d % max(L, 1)) >= L - window)[None, :]
    M = torch.cat([seq_mask, dep_mask], dim=1)
    Kc = torch.cat([K, Kd], dim=2)
    Vc = torch.cat([V, Vd], dim=2)
    S = torch.matmul(Qf, Kc.transpose(-1, -2)) * scale
    S = S.masked_fill(~M, float("-inf"))
    lse = torch.logsumexp(S, dim=-1)
    Of = torch.matmul(torch.softmax(S, dim=-1), Vc)
    O = Of.reshape(B, Hk, T, G, d).permute(0, 1, 3, 2, 4).reshape(B, Hq, T, d)
    LSE = lse.reshape(B, Hk, T, G).permute(0, 1, 3, 2).reshape(B, Hq, T)
    return O, LSE


# -------------------------------------- Algorithm 1 (online softmax), fp64 ----
def algorithm1(Q, K, V, Kd, Vd, block_q_tokens=3, block_k=5, block_d=7):
    """Fused online softmax over G-aligned query blocks, written from the
    pages' description: running (m, acc, o) in base 2; loop 1 over key blocks
    wholly before the block's first base-time index; loop 2 over the boundary
    blocks with the grouped causal mask; loop 3 over depth blocks in
    [t_start*L, t_end*L) with the depth matching mask; finally o / acc."""
    Q, K, V, Kd, Vd = (np.asarray(x, dtype=np.float64) for x in (Q, K, V, Kd, Vd))
    B, Hq, T, d = Q.shape
    Hk = K.shape[1]
    G = Hq // Hk
    L = Kd.shape[2] // T if T else 0
    c = LOG2E / math.sqrt(d)
    O = np.zeros_like(Q)
    LSE = np.zeros((B, Hq, T))
    BQ = block_q_tokens * G            # block size divisible by G
    for b in range(B):
        for hk in range(Hk):
            Qf = Q[b, hk * G:(hk + 1) * G].transpose(1, 0, 2).reshape(T * G, d)
            for r0 in range(0, T * G, BQ):
                r1 = min(r0 + BQ, T * G)
                rows = np.arange(r0, r1)
                tb = rows // G
                t_start, t_end = int(tb.min()), int(tb.max()) + 1
                m = np.full(r1 - r0, -np.inf)
                acc = np.zeros(r1 - r0)
                o = np.zeros((r1 - r0, d))

                def update(S, Vblk):
                    nonlocal m, acc, o
                    m_new = np.maximum(m, S.max(axis=1))
                    alpha = np.exp2(m - m_new)
                    P = np.exp2(S - m_new[:, None])
                    acc = acc * alpha + P.sum(axis=1)
                    o = o * alpha[:, None] + P @ Vblk
                    m = m_new

                # loop 1: unmasked key blocks, wholly before t_start
                j = 0
                while j + block_k <= t_start:
                    S = (Qf[r0:r1] @ K[b, hk, j:j + block_k].T) * c
                    update(S, V[b, hk, j:j + block_k])
                    j += block_k
                # loop 2: boundary blocks up to t_end, grouped causal mask
                while j < t_end:
                    je = min(j + block_k, T)
                    S = (Qf[r0:r1] @ K[b, hk, j:je].T) * c
                    ik = np.arange(j, je)
                    S = np.where(tb[:, None] >= ik[None, :], S, -np.inf)
                    update(S, V[b, hk, j:je])
                    j = je
                # loop 3: depth blocks of [t_start*L, t_end*L), matching mask
                jd = t_start * L
                while jd < t_end * L:
                    je = min(jd + block_d, t_end * L)
                    S = (Qf[r0:r1] @ Kd[b, hk, jd:je].T) * c
                    cols = np.arange(jd, je)
                    S = np.where(tb[:, None] == (cols // L)[None, :], S, -np.inf)
                    update(S, Vd[b, hk, jd:je])
                    jd = je
                out = o / acc[:, None]
                lse = (m + np.log2(acc)) / LOG2E
                for i, r in enumerate(rows):
                    t, g = divmod(int(r), G)
                    O[b, hk * G + g, t] = out[i]
                    LSE[b, hk * G + g, t] = lse[i]
    return O, LSE


# -------------------------------------------------------------------- pins ----
def _close(a, b, tol, what):
    a = np.asarray(a)
    b = np.asarray(b)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max |diff| = {err:.3e} > {tol:.1e}"


def pin_l0_is_causal_sdpa(lib):
    """L = 0 is causal softmax attention (library SDPA on repeat_interleaved
    K/V, fp64), with LSE from torch.logsumexp over the causal score matrix."""
    for (B, Hq, Hk, T, d, seed) in ((2, 4, 2, 13, 16, 1), (1, 6, 2, 9, 8, 2), (1, 3, 3, 1, 4, 3)):
        Q, K, V, _, _, _ = rand_case(B, Hq, Hk, T, d, 0, seed)
        O, LSE = oracle.fwd(Q, K, V, None, None, lib=lib)
        G = Hq // Hk
        Ke, Ve = K.repeat_interleave(G, dim=1), V.repeat_interleave(G, dim=1)
        ref = torch.nn.functional.scaled_dot_product_attention(Q, Ke, Ve, is_causal=True)
        S = (Q @ Ke.transpose(-1, -2)) / math.sqrt(d)
        S = S.masked_fill(torch.ones(T, T, dtype=torch.bool).triu(1), float("-inf"))
        _close(O, ref.numpy(), 1e-12, "O vs causal SDPA")
        _close(LSE, torch.logsumexp(S, -1).numpy(), 1e-12, "LSE vs logsumexp")


def pin_t1_self_plus_depth(lib):
    """T = 1: softmax over {key 0} plus the token's L depth keys (library SDPA,
    non-causal, over the concatenated key rows)."""
    B, Hq, Hk, T, d, L = 1, 4, 2, 1, 8, 5
    Q, K, V, Kd, Vd, _ = rand_case(B, Hq, Hk, T, d, L, 11)
    O, LSE = oracle.fwd(Q, K, V, Kd, Vd, lib=lib)
    G = Hq // Hk
    Kc = torch.cat([K, Kd], 2).repeat_interleave(G, dim=1)
    Vc = torch.cat([V, Vd], 2).repeat_interleave(G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, Kc, Vc)
    lse = torch.logsumexp((Q @ Kc.transpose(-1, -2)) / math.sqrt(d), -1)
    _close(O, ref.numpy(), 1e-12, "O at T=1")
    _close(LSE, lse.numpy(), 1e-12, "LSE at T=1")


def pin_dense_bruteforce(lib):
    """Against the dense [seq | depth] formulation with the full mask matrix
    in the pages' flattened index (includes G = 1, G = 3, ragged T)."""
    for (B, Hq, Hk, T, d, L, seed) in ((1, 4, 2, 11, 8, 3, 21), (2, 3, 1, 7, 4, 2, 22),
                                       (1, 2, 2, 6, 16, 1, 23), (1, 6, 2, 5, 8, 4, 24)):
        Q, K, V, Kd, Vd, _ = rand_case(B, Hq, Hk, T, d, L, seed)
        O, LSE = oracle.fwd(Q, K, V, Kd, Vd, lib=lib)
        Or, LSEr = dense_moda(Q, K, V, Kd, Vd)
        _close(O, Or.numpy(), 1e-12, "O vs dense")
        _close(LSE, LSEr.numpy(), 1e-12, "LSE vs dense")


def pin_algorithm1(lib):
    """Online softmax (Algorithm 1) equals the materialised oracle (the pages
    call it exact); several block sizes, ragged tails."""
    for (B, Hq, Hk, T, d, L, seed, bq, bk, bd) in ((1, 4, 2, 13, 8, 3, 31, 3, 5, 7),
                                                   (1, 8, 2, 10, 4, 6, 32, 2, 4, 5),
                                                   (1, 2, 2, 9, 8, 2, 33, 4, 3, 3)):
        Q, K, V, Kd, Vd, _ = rand_case(B, Hq, Hk, T, d, L, seed)
        O, LSE = oracle.fwd(Q, K, V, Kd, Vd, lib=lib)
        Oa, LSEa = algorithm1(Q, K, V, Kd, Vd, bq, bk, bd)
        _close(O, Oa, 1e-12, "O vs Algorithm 1")
        _close(LSE, LSEa, 1e-12, "LSE vs Algorithm 1")


def pin_zero_query_closed_form(lib):
    """Q = 0: every visible score is 0, so O[t] is the plain mean of the t+1
    sequence values and the L depth values of token t; LSE = ln(t+1+L)."""
    B, Hq, Hk, T, d, L = 1, 4, 2, 9, 8, 3
    _, K, V, Kd, Vd, _ = rand_case(B, Hq, Hk, T, d, L, 41)
    Q = torch.zeros(B, Hq, T, d, dtype=torch.float64)
    O, LSE = oracle.fwd(Q, K, V, Kd, Vd, lib=lib)
    G = Hq // Hk
    Vn, Vdn = V.numpy(), Vd.numpy().reshape(B, Hk, T, L, d)
    csum = np.cumsum(Vn, axis=2)
    for h in range(Hq):
        hk = h // G
        n = np.arange(1, T + 1) + L
        ref = (csum[0, hk] + Vdn[0, hk].sum(axis=1)) / n[:, None]
        _close(O[0, h], ref, 1e-12, "O with Q=0")
        _close(LSE[0, h], np.log(n), 1e-12, "LSE with Q=0")


def pin_depth_permutation(lib):
    """Permuting a token's L depth rows (same permutation on K_depth and
    V_depth) leaves O and LSE unchanged; permuting K_depth alone changes O."""
    B, Hq, Hk, T, d, L = 1, 4, 2, 8, 8, 5
    Q, K, V, Kd, Vd, _ = rand_case(B, Hq, Hk, T, d, L, 51)
    O, LSE = oracle.fwd(Q, K, V, Kd, Vd, lib=lib)
    rng = np.random.default_rng(51)
    Kp = Kd.reshape(B, Hk, T, L, d).clone()
    Vp = Vd.reshape(B, Hk, T, L, d).clone()
    for t in range(T):
        perm = torch.from_numpy(rng.permutation(L))
        Kp[:, :, t] = Kp[:, :, t, perm]
        Vp[:, :, t] = Vp[:, :, t, perm]
    O2, LSE2 = oracle.fwd(Q, K, V, Kp.reshape_as(Kd), Vp.reshape_as(Vd), lib=lib)
    _close(O2, O, 1e-12, "O after depth permutation")
    _close(LSE2, LSE, 1e-12, "LSE after depth permutation")
    O3, _ = oracle.fwd(Q, K, V, Kp.reshape_as(Kd), Vd, lib=lib)
    assert np.max(np.abs(O3 - O)) > 1e-3, "depth keys and values are not paired"


def pin_gqa_is_repeat_interleave(lib):
    """GQA equals MHA on repeat_interleaved K, V, K_depth, V_depth."""
    B, Hq, Hk, T, d, L = 2, 6, 2, 7, 8, 3
    Q, K, V, Kd, Vd, dO = rand_case(B, Hq, Hk, T, d, L, 61)
    G = Hq // Hk
    O, LSE = oracle.fwd(Q, K, V, Kd, Vd, lib=lib)
    ri = lambda x: x.repeat_interleave(G, dim=1)
    O2, LSE2 = oracle.fwd(Q, ri(K), ri(V), ri(Kd), ri(Vd), lib=lib)
    _close(O, O2, 1e-12, "GQA vs expanded MHA")
    _close(LSE, LSE2, 1e-12, "GQA LSE vs expanded MHA")
    # the per-KV-head gradients are the sums over the group of the MHA ones
    g1 = oracle.bwd(Q, K, V, Kd, Vd, dO, lib=lib)
    g2 = oracle.bwd(Q, ri(K), ri(V), ri(Kd), ri(Vd), dO, lib=lib)
    _close(g1[0], g2[0], 1e-11, "dQ GQA vs MHA")
    for a, b2, nm in ((g1[1], g2[1], "dK"), (g1[2], g2[2], "dV"),
                      (g1[3], g2[3], "dKd"), (g1[4], g2[4], "dVd")):
        red = b2.reshape(B, Hk, G, *b2.shape[2:]).sum(axis=2)
        _close(a, red, 1e-11, f"{nm} GQA vs group-summed MHA")


def pin_convexity(lib):
    """Each output coordinate lies within [min, max] of the values the row
    attends to (its sequence prefix and its own depth rows)."""
    B, Hq, Hk, T, d, L = 1, 2, 1, 10, 4, 3
    Q, K, V, Kd, Vd, _ = rand_case(B, Hq, Hk, T, d, L, 71)
    Q = Q * 3.0
    O, _ = oracle.fwd(Q, K, V, Kd, Vd, lib=lib)
    Vn, Vdn = V.numpy()[0, 0], Vd.numpy()[0, 0].reshape(T, L, d)
    for h in range(Hq):
        for t in range(T):
            vals = np.concatenate([Vn[:t + 1], Vdn[t]], axis=0)
            assert np.all(O[0, h, t] >= vals.min(0) - 1e-12)
            assert np.all(O[0, h, t] <= vals.max(0) + 1e-12)


def pin_bwd_autograd(lib):
    """Backward equals torch autograd through the dense formulation (fp64)."""
    for (B, Hq, Hk, T, d, L, seed) in ((1, 4, 2, 9, 8, 3, 81), (2, 3, 1, 6, 4, 2, 82),
                                       (1, 2, 2, 5, 8, 0, 83)):
        Q, K, V, Kd, Vd, dO = rand_case(B, Hq, Hk, T, d, L, seed)
        xs = [x.clone().requires_grad_(True) for x in (Q, K, V, Kd, Vd)]
        O, _ = dense_moda(*xs)
        grads = torch.autograd.grad((O * dO).sum(), xs, allow_unused=True)
        mine = oracle.bwd(Q, K, V, Kd, Vd, dO, lib=lib)
        for nm, a, g in zip(("dQ", "dK", "dV", "dKd", "dVd"), mine, grads):
            ref = np.zeros(a.shape) if g is None else g.numpy()
            _close(a, ref, 1e-11, f"{nm} vs autograd")


def pin_bwd_finite_differences(lib):
    """Central differences of f = <dO, O> along random directions match the
    oracle's gradients (fp64, eps = 1e-6)."""
    B, Hq, Hk, T, d, L = 1, 4, 2, 6, 8, 3
    Q, K, V, Kd, Vd, dO = rand_case(B, Hq, Hk, T, d, L, 91)
    base = [x.numpy() for x in (Q, K, V, Kd, Vd)]
    grads = oracle.bwd(*base, dO.numpy(), lib=lib)
    rng = np.random.default_rng(91)
    eps = 1e-6

    def f(args):
        O, _ = oracle.fwd(*args, lib=lib)
        return float(np.sum(O * dO.numpy()))

    for i, nm in enumerate(("Q", "K", "V", "Kd", "Vd")):
        u = rng.standard_normal(base[i].shape)
        plus = list(base)
        minus = list(base)
        plus[i] = base[i] + eps * u
        minus[i] = base[i] - eps * u
        fd = (f(plus) - f(minus)) / (2 * eps)
        an = float(np.sum(grads[i] * u))
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), f"d{nm}: fd {fd} vs {an}"


def pin_repack_definition(lib):
    """Layer-major [L,B,Hk,T,d] -> token-major [B,Hk,T*L,d]: row t*L + l of the
    output is layer l of token t (numpy transpose + reshape); bytewise."""
    L, B, Hk, T, d = 3, 2, 2, 5, 4
    src = np.arange(L * B * Hk * T * d, dtype=np.uint16).reshape(L, B, Hk, T, d)
    out = oracle.repack(src, B, Hk, T, d, L, lib=lib)
    ref = src.transpose(1, 2, 3, 0, 4).reshape(B, Hk, T * L, d)
    assert out.dtype == src.dtype and np.array_equal(out, ref), "repack permutation"


def pin_noncausal_l0_is_sdpa(lib):
    """Non-causal with L = 0 is plain softmax attention over all T keys
    (library SDPA without the causal mask, repeat_interleaved K/V)."""
    for (B, Hq, Hk, T, d, seed) in ((1, 4, 2, 11, 16, 101), (2, 3, 3, 6, 8, 102)):
        Q, K, V, _, _, _ = rand_case(B, Hq, Hk, T, d, 0, seed)
        O, LSE = oracle.fwd(Q, K, V, None, None, lib=lib, causal=False)
        G = Hq // Hk
        Ke, Ve = K.repeat_interleave(G, dim=1), V.repeat_interleave(G, dim=1)
        ref = torch.nn.functional.scaled_dot_product_attention(Q, Ke, Ve)
        lse = torch.logsumexp((Q @ Ke.transpose(-1, -2)) / math.sqrt(d), -1)
        _close(O, ref.numpy(), 1e-12, "non-causal O vs SDPA")
        _close(LSE, lse.numpy(), 1e-12, "non-causal LSE")


def pin_modes_dense_bruteforce(lib):
    """Non-causal and depth-window forward against the dense formulation."""
    for (causal, window, seed) in ((False, 0, 111), (True, 2, 112), (False, 3, 113), (True, 4, 114)):
        Q, K, V, Kd, Vd, _ = rand_case(1, 4, 2, 9, 8, 4, seed)
        O, LSE = oracle.fwd(Q, K, V, Kd, Vd, lib=lib, causal=causal, window=window)
        Or, LSEr = dense_moda(Q, K, V, Kd, Vd, causal=causal, window=window)
        _close(O, Or.numpy(), 1e-12, f"O causal={causal} window={window}")
        _close(LSE, LSEr.numpy(), 1e-12, f"LSE causal={causal} window={window}")


def pin_window_is_truncated_depth(lib):
    """A depth window of S equals the full-depth operator on depth tensors
    cut to each token's last S layers (L' = S)."""
    B, Hq, Hk, T, d, L, S = 2, 4, 2, 7, 8, 5, 2
    Q, K, V, Kd, Vd, _ = rand_case(B, Hq, Hk, T, d, L, 121)
    cut = lambda x: x.reshape(B, Hk, T, L, d)[:, :, :, L - S:].reshape(B, Hk, T * S, d)
    O, LSE = oracle.fwd(Q, K, V, Kd, Vd, lib=lib, window=S)
    O2, LSE2 = oracle.fwd(Q, K, V, cut(Kd), cut(Vd), lib=lib)
    _close(O, O2, 1e-12, "window O vs truncated depth")
    _close(LSE, LSE2, 1e-12, "window LSE vs truncated depth")
    g = oracle.bwd(Q, K, V, Kd, Vd, rand_case(B, Hq, Hk, T, d, L, 122)[5], lib=lib, window=S)
    g2 = oracle.bwd(Q, K, V, cut(Kd), cut(Vd), rand_case(B, Hq, Hk, T, d, L, 122)[5], lib=lib)
    for i, nm in ((0, "dQ"), (1, "dK"), (2, "dV")):
        _close(g[i], g2[i], 1e-11, f"window {nm}")
    full = g[3].reshape(B, Hk, T, L, d)
    _close(full[:, :, :, L - S:].reshape(B, Hk, T * S, d), g2[3], 1e-11, "window dKd")
    assert np.all(full[:, :, :, :L - S] == 0.0), "rows outside the window get zero gradient"


def pin_modes_bwd_autograd(lib):
    """Backward of the non-causal and windowed operator equals autograd
    through the dense formulation."""
    for (causal, window, seed) in ((False, 0, 131), (True, 2, 132), (False, 1, 133)):
        Q, K, V, Kd, Vd, dO = rand_case(1, 4, 2, 7, 8, 3, seed)
        xs = [x.clone().requires_grad_(True) for x in (Q, K, V, Kd, Vd)]
        O, _ = dense_moda(*xs, causal=causal, window=window)
        grads = torch.autograd.grad((O * dO).sum(), xs)
        mine = oracle.bwd(Q, K, V, Kd, Vd, dO, lib=lib, causal=causal, window=window)
        for nm, a, g in zip(("dQ", "dK", "dV", "dKd", "dVd"), mine, grads):
            _close(a, g.numpy(), 1e-11, f"{nm} causal={causal} window={window}")


def pin_decode_is_last_row(lib):
    """Decoding the newest token equals the last row of the full operator
    over the whole sequence (with and without a depth window)."""
    B, Hq, Hk, T, d, L = 2, 6, 2, 9, 8, 4
    Q, K, V, Kd, Vd, _ = rand_case(B, Hq, Hk, T, d, L, 141)
    last = lambda x: x.reshape(B, Hk, T, L, d)[:, :, T - 1]
    for window in (0, 3):
        O, LSE = oracle.fwd(Q, K, V, Kd, Vd, lib=lib, window=window)
        o, lse = oracle.decode(Q[:, :, T - 1], K, V, last(Kd), last(Vd), window=window, lib=lib)
        _close(o, O[:, :, T - 1], 1e-12, f"decode O window={window}")
        _close(lse, LSE[:, :, T - 1], 1e-12, f"decode LSE window={window}")


ALL_PINS = [pin_decode_is_last_row, pin_l0_is_causal_sdpa, pin_t1_self_plus_depth, pin_dense_bruteforce,
            pin_algorithm1, pin_zero_query_closed_form, pin_depth_permutation,
            pin_gqa_is_repeat_interleave, pin_convexity, pin_bwd_autograd,
            pin_bwd_finite_differences, pin_repack_definition, pin_noncausal_l0_is_sdpa,
            pin_modes_dense_bruteforce, pin_window_is_truncated_depth, pin_modes_bwd_autograd]


def pin_worked_example(lib):
    """The exact worked example (tests/golden): forward, LSE and all five
    gradients equal values derived by hand-checkable Fraction arithmetic
    from the definition, to 1e-12."""
    from worked_example import load
    x, e = load()
    O, LSE = oracle.fwd(x["Q"], x["K"], x["V"], x["Kd"], x["Vd"], lib=lib)
    _close(O, e["O"], 1e-12, "worked example O")
    _close(LSE, e["LSE"], 1e-12, "worked example LSE")
    grads = oracle.bwd(x["Q"], x["K"], x["V"], x["Kd"], x["Vd"], x["dO"], lib=lib)
    for name, got in zip(("dQ", "dK", "dV", "dKd", "dVd"), grads):
        _close(got, e[name], 1e-12, f"worked example {name}")


ALL_PINS.append(pin_worked_example)
