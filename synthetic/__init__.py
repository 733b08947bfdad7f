"""Seeded synthetic inputs shared by the tests, the bench and the oracle.

This module holds no arithmetic of the method: it only draws random tensors
with the shapes and value distributions of the workloads (activations with
channel outliers and spikes, Gaussian weights, Zipf-skewed expert routing).
The activation model stands in for the real-model activations of
Llama-3.1-8B, Qwen2.5-7B and Qwen3-30B-A3B that the SharQ evaluation uses;
the weights stand in for trained checkpoints (random init ~N(0, 0.02)).

All draws use numpy's PCG64 generator; values are drawn in float32 and rounded
to bfloat16 (round to nearest even) at the end.
"""
import numpy as np


def _to_bf16(x):
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def activations(seed, T, K, *, n_channels=None, channel_frac=0.005,
                channel_scale=(20.0, 60.0), spike_p=0.001, spike_mag=(8.0, 16.0),
                base="normal", student_nu=3.0):
    """Outlier activation model, float32 [T, K] holding bf16 values.

    1. base N(0,1) (or Student-t(nu) when base == "student_t");
    2. channel outliers: `n_channels` distinct columns (default
       round(channel_frac*K)) multiplied by U(channel_scale) (a fixed
       multiplier when the tuple has equal ends);
    3. spikes: each entry independently, with probability spike_p, replaced
       by +-U(spike_mag) with a fair sign.
    """
    g = rng(seed)
    if base == "normal":
        x = g.standard_normal((T, K), dtype=np.float32)
    elif base == "student_t":
        x = g.standard_t(student_nu, size=(T, K)).astype(np.float32)
    else:
        raise ValueError(base)
    if n_channels is None:
        n_channels = int(round(channel_frac * K))
    if n_channels > 0:
        ch = g.choice(K, size=n_channels, replace=False)
        lo, hi = channel_scale
        mult = g.uniform(lo, hi, size=n_channels).astype(np.float32) if hi > lo \
            else np.full(n_channels, lo, dtype=np.float32)
        x[:, ch] *= mult[None, :]
    if spike_p > 0:
        hit = g.random((T, K)) < spike_p
        mag = g.uniform(spike_mag[0], spike_mag[1], size=(T, K)).astype(np.float32)
        sgn = np.where(g.random((T, K)) < 0.5, -1.0, 1.0).astype(np.float32)
        x = np.where(hit, sgn * mag, x)
    return _to_bf16(x)


def weights(seed, K, D, std=0.02):
    """W in R^{K x D}, float32 holding bf16 values, ~N(0, std)."""
    g = rng(seed)
    return _to_bf16(g.standard_normal((K, D), dtype=np.float32) * np.float32(std))


def gamma(seed, K, lo=0.5, hi=1.5):
    """RMSNorm weight ~U(lo, hi) (bf16); lo == hi gives a constant."""
    if lo == hi:
        return _to_bf16(np.full(K, lo, dtype=np.float32))
    g = rng(seed)
    return _to_bf16(g.uniform(lo, hi, size=K).astype(np.float32))


def moe_routing(seed, T, n_experts=128, top_k=8, zipf_s=1.1):
    """Expert choice per token: expert popularity ~ rank^-s over a seeded
    permutation of the experts; each token draws top_k distinct experts
    without replacement.  Returns (token index per expert-sorted row int64
    [T*top_k], group offsets int64 [E+1])."""
    g = rng(seed)
    perm = g.permutation(n_experts)
    pop = np.empty(n_experts)
    pop[perm] = (np.arange(1, n_experts + 1, dtype=np.float64)) ** (-zipf_s)
    pop /= pop.sum()
    choice = np.empty((T, top_k), dtype=np.int64)
    for t in range(T):
        choice[t] = g.choice(n_experts, size=top_k, replace=False, p=pop)
    expert = choice.reshape(-1)
    token = np.repeat(np.arange(T, dtype=np.int64), top_k)
    order = np.argsort(expert, kind="stable")
    counts = np.bincount(expert, minlength=n_experts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    return token[order], offsets
