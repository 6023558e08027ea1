"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers; it holds none of the method's
arithmetic, so both the CUDA path's tests and the CPU oracle's tests take
their inputs from here.

The pages train Qwen3-0.6B on DCLM (Lighthouse review of "The Curse and
Blessing of Mean Bias in FP4-Quantized LLM Training", section 三 3.1); neither
the data nor trained activations are available, so these generators stand in
for them with the structure the pages describe: a rank-one column mean, a
low-rank spike and a Gaussian tail (section 二 2.1, the three-component
decomposition X = 1 mu^T + U_k S_k V_k^T + X_tail), a few "hot" channels with
a large mean, and a SwiGLU-style positive-mean input for the FFN
down-projection (section 二 2.2, stage II: E[phi(z)] > 0).

Every generator uses numpy's PCG64 with seed = 1000 * workload + tag, draws in
fp64 and rounds to the storage dtype (fp32, or bf16 with round to nearest
even).  N(a, s) means mean a and standard deviation s.
"""

import numpy as np

try:  # torch is only needed for the bf16 rounding and device copies
    import torch
except Exception:  # pragma: no cover
    torch = None


def rng_for(workload, tag):
    return np.random.Generator(np.random.PCG64(1000 * int(workload) + int(tag)))


def _orthonormal(rng, rows, k):
    q, _ = np.linalg.qr(rng.standard_normal((rows, k)))
    return q


def spiked_activations(rng, l, m, rank, s, n_hot, mu_std=0.5, hot_scale=20.0,
                       mean_scale=1.0):
    """X = mean_scale * 1 mu^T + U diag(s) V^T + N(0, 1), fp64 [l, m].

    mu_j ~ N(0, mu_std) with ``n_hot`` random channels multiplied by
    ``hot_scale``; U [l, rank] and V [m, rank] are orthonormalised Gaussians.
    """
    mu = rng.normal(0.0, mu_std, m)
    if n_hot:
        hot = rng.choice(m, size=n_hot, replace=False)
        mu[hot] *= hot_scale
    u = _orthonormal(rng, l, rank)
    v = _orthonormal(rng, m, rank)
    X = mean_scale * mu[None, :] + (u * np.asarray(s, dtype=np.float64)) @ v.T
    X += rng.standard_normal((l, m))
    return X


def swiglu_input(rng, l, m, loc=0.2):
    """silu(a) * b with a, b ~ N(loc, 1) i.i.d.: a positive-mean, heavy-tailed
    down-projection input."""
    a = rng.normal(loc, 1.0, (l, m))
    b = rng.normal(loc, 1.0, (l, m))
    return a / (1.0 + np.exp(-a)) * b


def output_gradient(rng, l, n, scale=1e-3, col_mean_std=0.3):
    """scale * (N(0, 1) + per-column mean ~ N(0, col_mean_std))."""
    cm = rng.normal(0.0, col_mean_std, n)
    return scale * (rng.standard_normal((l, n)) + cm[None, :])


def weight(rng, m, n):
    """W [m, n] ~ N(0, 1/sqrt(m)) (in-features m, out-features n)."""
    return rng.normal(0.0, 1.0 / np.sqrt(m), (m, n))


def planted_mean_columns(rng, l, mus, sigma=1.0):
    """Columns with planted means ``mus`` plus N(0, sigma) noise, fp64."""
    mus = np.asarray(mus, dtype=np.float64)
    return mus[None, :] + sigma * rng.standard_normal((l, mus.size))


# --------------------------------------------------------------------------
# storage rounding
# --------------------------------------------------------------------------
def to_f32(X):
    return np.ascontiguousarray(np.asarray(X, dtype=np.float32))


def to_bf16(X):
    """fp64/fp32 numpy -> torch.bfloat16 CPU tensor (round to nearest even)."""
    return torch.from_numpy(to_f32(X)).to(torch.bfloat16)


def bf16_as_f32(t):
    """torch.bfloat16 tensor -> exact fp32 numpy copy."""
    return t.float().cpu().numpy()


# --------------------------------------------------------------------------
# the workloads
# --------------------------------------------------------------------------
# Each linear: (name, l, m, n, activation kind).
WORKLOADS = {
    0: dict(name="tiny forward-only linear", l=256, m=128, n=256, dtype="f32"),
    1: dict(name="Qwen3-0.6B fused QKV projection, fwd+dgrad", l=8192, m=1024, n=4096,
            dtype="bf16"),
    2: dict(name="Qwen3-0.6B FFN gate/up + down, fwd+dgrad", l=16384, dtype="bf16",
            linears=[("gate_up", 1024, 6144), ("down", 3072, 1024)]),
    3: dict(name="mean-strength sweep, one linear", l=16384, m=2048, n=2048, dtype="bf16",
            mean_scales=[0.0, 0.5, 2.0, 8.0, 32.0]),
}


def workload0(seed_tag=0):
    """Tiny forward-only case: X fp32 [256, 128], W fp32 [128, 256]."""
    rng = rng_for(0, 1 + seed_tag)
    X = spiked_activations(rng, 256, 128, rank=2, s=(8.0, 4.0), n_hot=2)
    W = weight(rng_for(0, 2 + seed_tag), 128, 256)
    return to_f32(X), to_f32(W)


def workload1(l=8192, m=1024, n=4096, seed_tag=0):
    """QKV projection: X bf16 [l, m], W bf16 [m, n], dY bf16 [l, n]."""
    n_hot = int(round(0.01 * m))
    X = spiked_activations(rng_for(1, 1 + seed_tag), l, m, rank=4,
                           s=(16.0, 8.0, 6.0, 4.0), n_hot=n_hot)
    W = weight(rng_for(1, 2 + seed_tag), m, n)
    D = output_gradient(rng_for(1, 3 + seed_tag), l, n)
    return to_bf16(X), to_bf16(W), to_bf16(D)


def workload2_down(l=16384, m=3072, n=1024, seed_tag=0):
    X = swiglu_input(rng_for(2, 11 + seed_tag), l, m)
    W = weight(rng_for(2, 12 + seed_tag), m, n)
    D = output_gradient(rng_for(2, 13 + seed_tag), l, n)
    return to_bf16(X), to_bf16(W), to_bf16(D)


def workload3(c, l=16384, m=2048, n=2048, seed_tag=0):
    """Mean-strength sweep: X = c 1 mu^T (mu ~ N(0,1)) + rank-4 spike + N(0,1)."""
    X = spiked_activations(rng_for(3, 1 + seed_tag), l, m, rank=4,
                           s=(16.0, 8.0, 6.0, 4.0), n_hot=0, mu_std=1.0,
                           mean_scale=c)
    W = weight(rng_for(3, 2 + seed_tag), m, n)
    return to_bf16(X), to_bf16(W)


def moe_counts(E, tokens, top_k, seed=0, alpha=1.0):
    """Tokens routed to each of E experts when every token picks top_k
    distinct experts, drawn with expert popularities p ~ Dirichlet(alpha): a
    skewed load like a trained router's.  Returns a list of E ints summing to
    tokens * top_k."""
    rng = rng_for(4, 100 + seed)
    p = rng.dirichlet(np.full(E, alpha))
    counts = np.zeros(E, dtype=np.int64)
    for _ in range(tokens):
        counts[rng.choice(E, top_k, replace=False, p=p)] += 1
    return [int(c) for c in counts]


def workload_moe(E=64, tokens=4096, top_k=8, m=2048, n=1024, seed_tag=0):
    """A mixture-of-experts linear: the permuted activation buffer [l_cap, m]
    (expert e's tokens carry their own planted mean, spike and noise; rows of
    the 128-row padding are zero), the per-expert counts, the expert weights
    [E, m, n] and an output gradient in the same segments."""
    counts = moe_counts(E, tokens, top_k, seed_tag)
    rng = rng_for(5, 1 + seed_tag)
    offs, l_cap = [], 0
    for c in counts:
        offs.append(l_cap)
        l_cap += (c + 127) // 128 * 128
    X = np.zeros((l_cap, m))
    D = np.zeros((l_cap, n))
    for e, (o, c) in enumerate(zip(offs, counts)):
        if c:
            X[o:o + c] = spiked_activations(rng, c, m, rank=2, s=(8.0, 4.0), n_hot=m // 100,
                                            mean_scale=1.0 + (e % 4) / 2)
            D[o:o + c] = output_gradient(rng, c, n)
    W = np.stack([weight(rng, m, n) for _ in range(E)])
    return counts, to_bf16(X), to_bf16(W), to_bf16(D)
