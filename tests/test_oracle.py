"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: a special
case that reduces to a differently written rule (DeltaNet, Gated DeltaNet, pure
decay), a closed form, brute force over explicit transition matrices, or an
invariant of the recurrence.  Non-square states (dk != dv) are used wherever a
transposed operand could otherwise hide.

Which mistake each pin catches:
  test_deltanet_alpha_one          sign / placement of the erase and write terms
  test_gdn_scalar_gate             gate applied to the whole state, scalar case
  test_pure_decay_closed_form      dropped or mis-accumulated per-channel decay
  test_transition_product          order of decay and erase, transposes, beta
  test_exact_recall                output read from the post-update state, scale
  test_homogeneity                 a constant or bias term that should not exist
  test_split_sequence              state hand-off (resume from final_state)
  test_varlen_packing              sequence boundaries, zero-length sequences
  test_chunked_equals_token        the chunk algebra (WY / UT / substitution)
  test_l2norm_option               the fused L2Norm of q, k: per (token, head)
                                   row over dk, positive-scale invariant
  test_out_norm_gate_option        the output RMSNorm and gate: axis, eps,
                                   weight and gate placement
  test_backward_finite_differences every adjoint of kda_backward against
                                   central differences (varlen, initial state)
  test_backward_matches_autograd   the same against torch autograd of a plain
                                   recurrence, across the oracle's checkpoints
  test_backward_zero_adjoints_...  zero adjoints, the d_final_state default
  test_chunked_backward_equals_... the chunk-form adjoint (explicit inverse,
                                   the formulas the CUDA backward follows)
                                   against the token-form adjoint, C = 1..64
"""
import numpy as np
import pytest

import oracle
from oracle import chunked

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def rand_inputs(rng, B, T, H, dk, dv, unit_k=True, beta=None, g=None):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_k:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    if beta is None:
        beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    if g is None:
        g = -np.exp(rng.uniform(-5.0, -1.0, (B, T, H, dk)))
    return q, k, v, g, beta


# ---------------------------------------------------------------- O1
def test_deltanet_alpha_one():
    """alpha == 1 (log_alpha == 0): KDA is the delta rule.  Independent rule,
    written as on "深度解读报告" 2.2: read the value currently stored under the
    key, remove it along the key, write the new value (scaled by beta)."""
    rng = np.random.default_rng(1)
    B, T, H, dk, dv = 2, 13, 2, 5, 3
    q, k, v, _, beta = rand_inputs(rng, B, T, H, dk, dv)
    g = np.zeros((B, T, H, dk))
    s0 = rng.standard_normal((B, H, dk, dv))
    out, fs = oracle.kda_forward(q, k, v, g, beta, initial_state=s0, scale=0.7)
    for b in range(B):
        for h in range(H):
            S = s0[b, h].copy()
            for t in range(T):
                kt, vt = k[b, t, h], v[b, t, h]
                stored = np.einsum("cj,c->j", S, kt)
                S = S - beta[b, t, h] * np.outer(kt, stored) + beta[b, t, h] * np.outer(kt, vt)
                np.testing.assert_allclose(out[b, t, h], 0.7 * np.einsum("cj,c->j", S, q[b, t, h]),
                                           rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(fs[b, h], S, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- O2
def test_gdn_scalar_gate():
    """alpha constant over channels: KDA is Gated DeltaNet,
    S_t = (I - beta k k^T) alpha_t S_{t-1} + beta k v^T (zhaixingw.cn ai-news/151,
    the Gated DeltaNet formula), with the dk x dk matrix formed explicitly."""
    rng = np.random.default_rng(2)
    B, T, H, dk, dv = 1, 17, 3, 4, 6
    q, k, v, _, beta = rand_inputs(rng, B, T, H, dk, dv)
    a = rng.uniform(0.5, 1.0, (B, T, H))
    g = np.repeat(np.log(a)[..., None], dk, axis=-1)
    s0 = rng.standard_normal((B, H, dk, dv))
    out, fs = oracle.kda_forward(q, k, v, g, beta, initial_state=s0, scale=1.3)
    for h in range(H):
        S = s0[0, h].copy()
        for t in range(T):
            kt = k[0, t, h]
            E = np.eye(dk) - beta[0, t, h] * np.outer(kt, kt)
            S = E @ (a[0, t, h] * S) + beta[0, t, h] * np.outer(kt, v[0, t, h])
            np.testing.assert_allclose(out[0, t, h], 1.3 * S.T @ q[0, t, h], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(fs[0, h], S, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- O3
def test_pure_decay_closed_form():
    """beta == 0: no erase and no write, only per-channel multiplicative decay
    ("深度解读报告" 2.3, the Mamba2-like case).  Closed form with a non-zero
    initial state: S_t = Diag(exp(sum_{i<=t} g_i)) S_0, o_t = scale S_t^T q_t."""
    rng = np.random.default_rng(3)
    B, T, H, dk, dv = 2, 40, 2, 6, 4
    q, k, v, g, _ = rand_inputs(rng, B, T, H, dk, dv)
    beta = np.zeros((B, T, H))
    s0 = rng.standard_normal((B, H, dk, dv))
    out, fs = oracle.kda_forward(q, k, v, g, beta, initial_state=s0, scale=0.5)
    G = np.cumsum(g, axis=1)  # [B, T, H, dk]
    for b in range(B):
        for h in range(H):
            for t in range(T):
                St = np.exp(G[b, t, h])[:, None] * s0[b, h]
                np.testing.assert_allclose(out[b, t, h], 0.5 * St.T @ q[b, t, h],
                                           rtol=1e-11, atol=1e-13)
            np.testing.assert_allclose(fs[b, h], np.exp(G[b, -1, h])[:, None] * s0[b, h],
                                       rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------- O4
@pytest.mark.parametrize("dk,dv,T", [(3, 2, 8), (4, 5, 7), (2, 2, 1)])
def test_transition_product(dk, dv, T):
    """Brute force over the unified recurrent form ("深度解读报告" 2.4): with the
    transition M_t = (I - beta_t k_t k_t^T) Diag(alpha_t),
        S_t = M_t ... M_1 S_0 + sum_{i<=t} (M_t ... M_{i+1}) beta_i k_i v_i^T,
    every matrix formed explicitly and multiplied in that order."""
    rng = np.random.default_rng(10 * dk + dv)
    q, k, v, g, beta = rand_inputs(rng, 1, T, 1, dk, dv, unit_k=False)
    s0 = rng.standard_normal((1, 1, dk, dv))
    out, fs = oracle.kda_forward(q, k, v, g, beta, initial_state=s0, scale=0.9)
    M = [(np.eye(dk) - beta[0, t, 0] * np.outer(k[0, t, 0], k[0, t, 0])) @ np.diag(np.exp(g[0, t, 0]))
         for t in range(T)]
    for t in range(T):
        prod = np.eye(dk)
        for j in range(t, -1, -1):
            prod = prod @ M[j]
        St = prod @ s0[0, 0]
        for i in range(t + 1):
            P = np.eye(dk)
            for j in range(t, i, -1):
                P = P @ M[j]
            St = St + P @ (beta[0, i, 0] * np.outer(k[0, i, 0], v[0, i, 0]))
        np.testing.assert_allclose(out[0, t, 0], 0.9 * St.T @ q[0, t, 0], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(fs[0, 0], St, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- O6
def test_exact_recall():
    """beta = 1 and a unit key: after the update the state returns exactly the
    value just written under that key, whatever was stored before and whatever
    the gate, so with q_t = k_t the output is scale * v_t."""
    rng = np.random.default_rng(6)
    B, T, H, dk, dv = 1, 30, 2, 8, 5
    _, k, v, g, _ = rand_inputs(rng, B, T, H, dk, dv)
    beta = np.ones((B, T, H))
    s0 = rng.standard_normal((B, H, dk, dv))
    out, _ = oracle.kda_forward(k, k, v, g, beta, initial_state=s0, scale=0.25)
    np.testing.assert_allclose(out, 0.25 * v, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- O7
def test_homogeneity():
    """The recurrence is linear in (S_0, V) jointly and in q: scaling S_0 and v
    by c scales out and S_T by c; scaling q by c scales out by c."""
    rng = np.random.default_rng(7)
    B, T, H, dk, dv = 1, 25, 2, 6, 3
    q, k, v, g, beta = rand_inputs(rng, B, T, H, dk, dv)
    s0 = rng.standard_normal((B, H, dk, dv))
    o1, f1 = oracle.kda_forward(q, k, v, g, beta, initial_state=s0)
    o2, f2 = oracle.kda_forward(q, k, -2.5 * v, g, beta, initial_state=-2.5 * s0)
    o3, _ = oracle.kda_forward(3.0 * q, k, v, g, beta, initial_state=s0)
    np.testing.assert_allclose(o2, -2.5 * o1, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(f2, -2.5 * f1, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(o3, 3.0 * o1, rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------- O8
def test_split_sequence():
    """Running tokens [0, t) and feeding the final state into [t, T) equals one
    run over [0, T): the fixed-size state is the whole carried history."""
    rng = np.random.default_rng(8)
    B, T, H, dk, dv = 2, 37, 2, 5, 4
    q, k, v, g, beta = rand_inputs(rng, B, T, H, dk, dv)
    s0 = rng.standard_normal((B, H, dk, dv))
    o, f = oracle.kda_forward(q, k, v, g, beta, initial_state=s0)
    for t in (1, 16, 36):
        oa, fa = oracle.kda_forward(q[:, :t], k[:, :t], v[:, :t], g[:, :t], beta[:, :t],
                                    initial_state=s0)
        ob, fb = oracle.kda_forward(q[:, t:], k[:, t:], v[:, t:], g[:, t:], beta[:, t:],
                                    initial_state=fa)
        np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(fb, f, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- O9
def test_varlen_packing():
    """Packing sequences into one stream with cu_seqlens equals running each
    separately; a zero-length sequence passes its initial state through."""
    rng = np.random.default_rng(9)
    lengths = [5, 0, 12, 1, 7]
    H, dk, dv = 2, 4, 3
    Ttot = sum(lengths)
    q, k, v, g, beta = rand_inputs(rng, 1, Ttot, H, dk, dv)
    s0 = rng.standard_normal((len(lengths), H, dk, dv))
    cu = np.cumsum([0] + lengths)
    o, f = oracle.kda_forward(q, k, v, g, beta, initial_state=s0, cu_seqlens=cu)
    for n, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        on, fn = oracle.kda_forward(q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b], beta[:, a:b],
                                    initial_state=s0[n:n + 1])
        np.testing.assert_allclose(o[:, a:b], on, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(f[n], fn[0], rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(f[1], s0[1])


def test_single_token_from_zero():
    """T = 1 from a zero state: S_1 = beta k v^T and o = scale beta (q.k) v."""
    rng = np.random.default_rng(11)
    q, k, v, g, beta = rand_inputs(rng, 1, 1, 1, 7, 3)
    out, fs = oracle.kda_forward(q, k, v, g, beta, scale=0.3)
    b = beta[0, 0, 0]
    np.testing.assert_allclose(fs[0, 0], b * np.outer(k[0, 0, 0], v[0, 0, 0]), rtol=1e-14)
    np.testing.assert_allclose(out[0, 0, 0], 0.3 * b * (q[0, 0, 0] @ k[0, 0, 0]) * v[0, 0, 0],
                               rtol=1e-13)


def test_default_scale_and_bad_args():
    rng = np.random.default_rng(12)
    q, k, v, g, beta = rand_inputs(rng, 1, 4, 1, 16, 2)
    o1, _ = oracle.kda_forward(q, k, v, g, beta)
    o2, _ = oracle.kda_forward(q, k, v, g, beta, scale=0.25)
    np.testing.assert_allclose(o1, o2, rtol=1e-15)
    with pytest.raises(ValueError):
        oracle.kda_forward(q, k, v, g, beta, cu_seqlens=[0, 2, 3])  # last != T


# ---------------------------------------------------------------- O5
@pytest.mark.parametrize("C", [1, 2, 3, 16, 64])
def test_chunked_equals_token(C):
    """The chunk algorithm equals the token recurrence for any chunk length,
    including a partial last chunk (T not a multiple of C) and packed
    sequences."""
    rng = np.random.default_rng(100 + C)
    lengths = [70, 1, 64, 0, 129]
    H, dk, dv = 2, 8, 6
    q, k, v, g, beta = rand_inputs(rng, 1, sum(lengths), H, dk, dv)
    s0 = 0.1 * rng.standard_normal((len(lengths), H, dk, dv))
    cu = np.cumsum([0] + lengths)
    o_ref, f_ref = oracle.kda_forward(q, k, v, g, beta, initial_state=s0, cu_seqlens=cu)
    o, f = chunked.chunked_forward(q, k, v, g, beta, initial_state=s0, cu_seqlens=cu, chunk=C)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(f, f_ref, rtol=1e-10, atol=1e-12)


def test_chunk_intermediates_consistent():
    """Inside one chunk: the rows of U solve the unrolled recurrence
    (I + A) U = Diag(beta)(V - Kt S0), computed here from the token loop's own
    erase coefficients u_r = beta_r (v_r - S_bar_r^T k_r)."""
    rng = np.random.default_rng(13)
    L, dk, dv = 9, 5, 4
    q, k, v, g, beta = rand_inputs(rng, 1, L, 1, dk, dv)
    S0 = rng.standard_normal((dk, dv))
    r = chunked.chunk_step(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], beta[0, :, 0], S0, 1.0)
    S = S0.copy()
    for t in range(L):
        S = np.exp(g[0, t, 0])[:, None] * S
        u = beta[0, t, 0] * (v[0, t, 0] - S.T @ k[0, t, 0])
        np.testing.assert_allclose(r["U"][t], u, rtol=1e-11, atol=1e-12)
        S = S + np.outer(k[0, t, 0], u)
    np.testing.assert_allclose(r["S"], S, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- L2Norm option
def test_l2norm_option():
    """With l2norm_qk the result depends on each q and k row only through its
    direction: (1) rows that are already unit vectors give exactly the plain
    result; (2) scaling every (token, head) row of q and of k by its own
    positive factor changes nothing (a normalisation over any other axis, or
    none, would not cancel per-row factors); (3) a zero key row stays zero
    (the 1e-6 floor), as in the plain call."""
    rng = np.random.default_rng(11)
    B, T, H, dk, dv = 2, 21, 3, 8, 5
    q, k, v, g, beta = rand_inputs(rng, B, T, H, dk, dv)       # unit rows
    s0 = rng.standard_normal((B, H, dk, dv))
    o_plain, f_plain = oracle.kda_forward(q, k, v, g, beta, initial_state=s0)
    o1, f1 = oracle.kda_forward(q, k, v, g, beta, initial_state=s0, l2norm_qk=True)
    np.testing.assert_allclose(o1, o_plain, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(f1, f_plain, rtol=1e-13, atol=1e-14)
    cq = np.exp(rng.uniform(-2.3, 2.3, (B, T, H, 1)))
    ck = np.exp(rng.uniform(-2.3, 2.3, (B, T, H, 1)))
    o2, f2 = oracle.kda_forward(cq * q, ck * k, v, g, beta, initial_state=s0, l2norm_qk=True)
    np.testing.assert_allclose(o2, o_plain, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(f2, f_plain, rtol=1e-11, atol=1e-12)
    kz = k.copy()
    kz[1, 7, 2] = 0.0
    o3, f3 = oracle.kda_forward(q, kz, v, g, beta, initial_state=s0, l2norm_qk=True)
    o4, f4 = oracle.kda_forward(q, kz, v, g, beta, initial_state=s0)
    np.testing.assert_allclose(o3, o4, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(f3, f4, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- raw gate
def test_raw_gate_option():
    """With raw_gate the log_alpha argument is the gate's pre-activation z
    and the decay is log sigmoid(z): (1) feeding z = logit(alpha) of a gate
    alpha reproduces the plain run with log alpha (the activation inverts
    the logit); (2) the log-gate equals torch's fp64 logsigmoid, a library
    routine, over [-60, 60] (no overflow at either end); (3) z = 0 halves the
    state every token (alpha = 1/2 exactly) in the pure-decay case."""
    import torch
    rng = np.random.default_rng(13)
    B, T, H, dk, dv = 2, 19, 3, 6, 5
    q, k, v, g, beta = rand_inputs(rng, B, T, H, dk, dv)
    s0 = rng.standard_normal((B, H, dk, dv))
    alpha = np.exp(g)
    z = np.log(alpha) - np.log1p(-alpha)
    o_plain, f_plain = oracle.kda_forward(q, k, v, g, beta, initial_state=s0)
    o_raw, f_raw = oracle.kda_forward(q, k, v, z, beta, initial_state=s0, raw_gate=True)
    np.testing.assert_allclose(o_raw, o_plain, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(f_raw, f_plain, rtol=1e-11, atol=1e-13)
    zz = np.linspace(-60.0, 60.0, 2001)
    ref = torch.nn.functional.logsigmoid(torch.from_numpy(zz)).numpy()
    np.testing.assert_allclose(oracle.log_sigmoid(zz), ref, rtol=1e-14, atol=1e-300)
    _, f_half = oracle.kda_forward(q, k, v, np.zeros_like(g), np.zeros_like(beta),
                                   initial_state=s0, raw_gate=True)
    np.testing.assert_allclose(f_half, s0 * 0.5 ** T, rtol=1e-13)


# ---------------------------------------------------------------- output RMSNorm + gate
def test_out_norm_gate_option():
    """The output epilogue takes each (token, head) row over dv: (1) with a
    saturated gate and unit weight every row's mean square is ms / (ms + eps)
    for the plain output's ms; (2) a zero pre-activation halves it exactly;
    (3) the weight scales channel j by w_j; (4) scaling v and S_0 by c > 0
    scales the plain output by c and, with a negligible eps, leaves the
    normalised one as it was."""
    rng = np.random.default_rng(12)
    B, T, H, dk, dv = 2, 17, 3, 6, 8
    q, k, v, g, beta = rand_inputs(rng, B, T, H, dk, dv)
    s0 = rng.standard_normal((B, H, dk, dv))
    o, _ = oracle.kda_forward(q, k, v, g, beta, initial_state=s0)
    eps = 1e-6
    ones = np.ones(dv)
    big = np.full(o.shape, 40.0)
    o1, f1 = oracle.kda_forward(q, k, v, g, beta, initial_state=s0, out_gate=big,
                                out_weight=ones, out_eps=eps)
    ms = np.mean(o * o, axis=-1)
    np.testing.assert_allclose(np.mean(o1 * o1, axis=-1), ms / (ms + eps), rtol=1e-12)
    _, f_plain = oracle.kda_forward(q, k, v, g, beta, initial_state=s0)
    np.testing.assert_array_equal(f1, f_plain)
    o2, _ = oracle.kda_forward(q, k, v, g, beta, initial_state=s0, out_gate=np.zeros(o.shape),
                               out_weight=ones, out_eps=eps)
    np.testing.assert_allclose(o2, 0.5 * o1, rtol=1e-13, atol=1e-15)
    w = rng.uniform(0.5, 2.0, dv)
    o3, _ = oracle.kda_forward(q, k, v, g, beta, initial_state=s0, out_gate=big,
                               out_weight=w, out_eps=eps)
    np.testing.assert_allclose(o3, o1 * w, rtol=1e-13, atol=1e-15)
    tiny = 1e-30
    o5, _ = oracle.kda_forward(q, k, v, g, beta, initial_state=s0, out_gate=big,
                               out_weight=ones, out_eps=tiny)
    o4, _ = oracle.kda_forward(q, k, 3.0 * v, g, beta, initial_state=3.0 * s0, out_gate=big,
                               out_weight=ones, out_eps=tiny)
    np.testing.assert_allclose(o4, o5, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- backward
#
# kda_backward is pinned two independent ways: central finite differences of
# the forward oracle (which catch a wrong sign, a dropped term or a
# transposed product in any of the six adjoints), and reverse-mode automatic
# differentiation of a plain torch fp64 recurrence.  T > 32 so that the
# oracle's block checkpointing (32 tokens) is crossed; varlen packing with a
# zero-length and a one-token sequence covers the chain boundaries.

def _loss_weights(rng, B, T, H, N, dk, dv):
    return rng.standard_normal((B, T, H, dv)), rng.standard_normal((N, H, dk, dv))


def test_backward_finite_differences():
    rng = np.random.default_rng(71)
    B, T, H, dk, dv = 1, 41, 1, 3, 2
    q, k, v, g, b = rand_inputs(rng, B, T, H, dk, dv)
    cu = np.array([0, 17, 17, 18, 41], dtype=np.int64)
    N = 4
    s0 = rng.standard_normal((N, H, dk, dv))
    Wo, Ws = _loss_weights(rng, B, T, H, N, dk, dv)

    def loss(*a):
        o, f = oracle.kda_forward(*a[:5], initial_state=a[5], cu_seqlens=cu, nthreads=1)
        return float((o * Wo).sum() + (f * Ws).sum())

    args = [q, k, v, g, b, s0]
    grads = oracle.kda_backward(q, k, v, g, b, Wo, initial_state=s0, d_final_state=Ws,
                                cu_seqlens=cu, nthreads=1)
    eps = 1e-6
    for ai, (a, gr) in enumerate(zip(args, grads)):
        assert gr.shape == a.shape
        fd = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            ap = [x.copy() for x in args]
            am = [x.copy() for x in args]
            ap[ai][idx] += eps
            am[ai][idx] -= eps
            fd[idx] = (loss(*ap) - loss(*am)) / (2 * eps)
        np.testing.assert_allclose(gr, fd, rtol=1e-6, atol=1e-7, err_msg=f"argument {ai}")


def _torch_recurrence(q, k, v, g, b, s0, cu, scale):
    """Plain token recurrence in torch fp64, written for autograd."""
    import torch
    outs, finals = [], []
    H = q.shape[2]
    for n in range(len(cu) - 1):
        for h in range(H):
            S = s0[n, h]
            for t in range(int(cu[n]), int(cu[n + 1])):
                S = torch.exp(g[0, t, h])[:, None] * S
                u = b[0, t, h] * (v[0, t, h] - S.T @ k[0, t, h])
                S = S + torch.outer(k[0, t, h], u)
                outs.append(((t, h), scale * (S.T @ q[0, t, h])))
            finals.append(S)
    return outs, finals


def test_backward_matches_autograd():
    import torch
    rng = np.random.default_rng(72)
    B, T, H, dk, dv = 1, 70, 2, 8, 5
    q, k, v, g, b = rand_inputs(rng, B, T, H, dk, dv, unit_k=False)
    cu = np.array([0, 33, 33, 70], dtype=np.int64)
    N = 3
    s0 = rng.standard_normal((N, H, dk, dv))
    Wo, Ws = _loss_weights(rng, B, T, H, N, dk, dv)
    scale = 0.37
    ts = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v, g, b, s0)]
    outs, finals = _torch_recurrence(*ts, cu, scale)
    Wo_t = torch.tensor(Wo)
    Ws_t = torch.tensor(Ws).reshape(N * H, dk, dv)
    loss = sum((o * Wo_t[0, t, h]).sum() for (t, h), o in outs)
    loss = loss + sum((f * Ws_t[i]).sum() for i, f in enumerate(finals))
    loss.backward()
    grads = oracle.kda_backward(q, k, v, g, b, Wo, initial_state=s0, d_final_state=Ws,
                                cu_seqlens=cu, scale=scale)
    for ai, (t, gr) in enumerate(zip(ts, grads)):
        np.testing.assert_allclose(gr, t.grad.numpy(), rtol=1e-9, atol=1e-11,
                                   err_msg=f"argument {ai}")


def test_backward_zero_adjoints_and_defaults():
    # no output adjoint and no final-state adjoint: every gradient is zero;
    # d_final_state=None means a zero adjoint of the final state
    rng = np.random.default_rng(73)
    q, k, v, g, b = rand_inputs(rng, 2, 9, 1, 4, 3)
    zeros = np.zeros((2, 9, 1, 3))
    for gr in oracle.kda_backward(q, k, v, g, b, zeros):
        assert not np.any(gr)
    do = rng.standard_normal((2, 9, 1, 3))
    a = oracle.kda_backward(q, k, v, g, b, do)
    c = oracle.kda_backward(q, k, v, g, b, do, d_final_state=np.zeros((2, 1, 4, 3)))
    for x, y in zip(a, c):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("C", [1, 3, 16, 64])
def test_chunked_backward_equals_token_backward(C):
    # the chunk-form adjoint (the algebra the CUDA backward implements) against
    # the token-form adjoint, packed sequences with a zero-length and a
    # one-token sequence, ragged chunks
    rng = np.random.default_rng(80 + C)
    B, T, H, dk, dv = 1, 45, 2, 6, 5
    q, k, v, g, b = rand_inputs(rng, B, T, H, dk, dv, unit_k=False)
    cu = np.array([0, 20, 20, 21, 45], dtype=np.int64)
    N = 4
    s0 = rng.standard_normal((N, H, dk, dv))
    do = rng.standard_normal((B, T, H, dv))
    dfs = rng.standard_normal((N, H, dk, dv))
    ref = oracle.kda_backward(q, k, v, g, b, do, initial_state=s0, d_final_state=dfs,
                              cu_seqlens=cu, scale=0.3)
    got = chunked.chunked_backward(q, k, v, g, b, do, initial_state=s0, d_final_state=dfs,
                                   cu_seqlens=cu, scale=0.3, chunk=C)
    for i, (a, r) in enumerate(zip(got, ref)):
        np.testing.assert_allclose(a, r, rtol=1e-10, atol=1e-12, err_msg=f"gradient {i}")
