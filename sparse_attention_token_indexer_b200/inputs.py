"""Seeded synthetic inputs shaped like the indexer workloads of the ADIndex paper.

This module only draws random numbers and prepares operand codes; it holds none of the
indexer's arithmetic, so both the CUDA path and the fp64 oracle can consume what it makes.
The paper measures on LongBench / RULER activations of DeepSeek-V3.2, which are not
available; these generators stand in for them with the same shapes (H_I = 64 indexer heads,
d = 128, K = 2048, contexts up to 256K) and with neighbouring queries that share Top-K keys.

Every generator takes a ``seed`` and a ``device``; torch's generator on that device is the
only source of randomness (the same seed on CPU and CUDA gives different but equally valid
draws, and each test compares the two sides on the very same tensors).
"""

import math

import torch

E4M3_MAX = 448.0


def _gen(seed, device):
    return torch.Generator(device=device).manual_seed(int(seed))


def _randn(gen, shape, device, scale=1.0):
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32) * scale


# ---------------------------------------------------------------------------------------
# FP8 input preparation (outside any timed region)
# ---------------------------------------------------------------------------------------

def quantize_e4m3_rows(x):
    """Per-row FP8-e4m3 codes: scale = amax(row) / 448 (1 for an all-zero row),
    code = round-to-nearest-even(x / scale) saturated to +-448.

    ``x`` [R, ...] float -> (codes uint8 [R, ...], scale float32 [R]).
    """
    xf = x.float()
    amax = xf.reshape(xf.shape[0], -1).abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = xf / scale.reshape((-1,) + (1,) * (xf.ndim - 1))
    codes = y.clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()


def as_operands(q, k, dtype):
    """bf16 tensors, or e4m3 codes + per-token scales, for q [T, H, d] and k [S, d]."""
    if dtype == "bf16":
        return dict(q=q.to(torch.bfloat16).contiguous(), q_scale=None,
                    k=k.to(torch.bfloat16).contiguous(), k_scale=None)
    if dtype == "e4m3":
        qc, qs = quantize_e4m3_rows(q)
        kc, ks = quantize_e4m3_rows(k)
        return dict(q=qc, q_scale=qs, k=kc, k_scale=ks)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------------------

def tiny_prefill(seed=0, device="cpu", T=1024, H=4, d=64, K=64):
    """Small causal prefill: q, k ~ N(0,1)/sqrt(d) in bf16, gates w ~ U(0,1)."""
    g = _gen(seed, device)
    q = _randn(g, (T, H, d), device, 1.0 / math.sqrt(d))
    k = _randn(g, (T, d), device, 1.0 / math.sqrt(d))
    w = torch.rand(T, H, generator=g, device=device, dtype=torch.float32)
    ops = as_operands(q, k, "bf16")
    ops.update(w=w, T=T, H=H, d=d, S=T, K=K, q_pos0=0, dtype="bf16")
    return ops


class AnchorStructure:
    """Keys and queries organised around shared anchor directions.

    keys:    S positions of N(0, I)/sqrt(d) noise; ``n_anchor`` unit directions u_m are each
             planted at ``copies`` distinct random positions as beta * u_m + sigma * noise.
    queries: token t carries two anchors (m1, m2) that change one at a time every ``block``
             tokens, plus a slowly drifting shared component eta_t and per-head noise:
             q[t, j] = gamma (u_m1 + u_m2) + rho eta_t + eps n_{t,j}.
             Neighbouring queries therefore share most of their Top-K keys.
    """

    def __init__(self, d, seed, device, n_anchor=256, copies=32, beta=1.0, sigma=0.5,
                 gamma=1.0, rho=0.5, eps=0.5, block=64):
        self.d, self.device = d, device
        self.n_anchor, self.copies = n_anchor, copies
        self.beta, self.sigma, self.gamma, self.rho, self.eps = beta, sigma, gamma, rho, eps
        self.block = block
        self.g = _gen(seed, device)
        u = _randn(self.g, (n_anchor, d), device)
        self.u = u / u.norm(dim=1, keepdim=True)

    def keys(self, S):
        d = self.d
        k = _randn(self.g, (S, d), self.device, 1.0 / math.sqrt(d))
        copies = min(self.copies, S // self.n_anchor)
        if copies > 0:
            n_plant = self.n_anchor * copies
            where = torch.randperm(S, generator=self.g, device=self.device)[:n_plant]
            which = torch.arange(self.n_anchor, device=self.device).repeat_interleave(copies)
            k[where] = self.beta * self.u[which] + self.sigma * k[where]
        return k

    def queries(self, T, H, pos0=0):
        d, dev, blk = self.d, self.device, self.block
        nb = (pos0 + T) // blk + 3
        ids = torch.randint(self.n_anchor, (nb,), generator=self.g, device=dev)
        coarse = _randn(self.g, (nb, d), dev, 1.0 / math.sqrt(d))
        pos = torch.arange(pos0, pos0 + T, device=dev)
        b = pos // blk
        frac = ((pos % blk).float() / blk).unsqueeze(1)
        eta = (1 - frac) * coarse[b] + frac * coarse[b + 1]
        base = self.gamma * (self.u[ids[b]] + self.u[ids[b + 1]]) + self.rho * eta
        noise = _randn(self.g, (T, H, d), dev, self.eps / math.sqrt(d))
        return base.unsqueeze(1) + noise

    def gates(self, T, H):
        return torch.rand(T, H, generator=self.g, device=self.device, dtype=torch.float32) / H


def anchor_prefill(T, H=64, d=128, K=2048, seed=1, device="cpu", dtype="bf16", S=None,
                   q_pos0=None):
    """Flat causal prefill on anchor-structured data.

    Keys cover positions 0..S-1 (S = T by default); the T query rows sit at positions
    q_pos0 .. q_pos0+T-1 (q_pos0 = S - T by default, i.e. the queries are the last T tokens).
    """
    S = T if S is None else S
    q_pos0 = S - T if q_pos0 is None else q_pos0
    st = AnchorStructure(d, seed, device)
    k = st.keys(S)
    q = st.queries(T, H, pos0=q_pos0)
    w = st.gates(T, H)
    ops = as_operands(q, k, dtype)
    ops.update(w=w, T=T, H=H, d=d, S=S, K=K, q_pos0=q_pos0, dtype=dtype)
    return ops


def mean_pool_group_queries(q, w, G, Hg):
    """Training-free group query: head j of group g is the mean over the G members of head j,
    for the first Hg heads; the group gate is the member mean of those heads' gates.

    q [T, H, d] (any float dtype), w [T, H] -> qbar [T // G, Hg, d] float32, wbar [T // G, Hg].
    """
    T = q.shape[0]
    ng = T // G
    qb = q[: ng * G, :Hg].float().reshape(ng, G, Hg, -1).mean(dim=1)
    wb = w[: ng * G, :Hg].float().reshape(ng, G, Hg).mean(dim=1)
    return qb.contiguous(), wb.contiguous()


def group_prefill(T, H=64, d=128, K=2048, G=64, B=8192, Hg=16, seed=2, device="cpu",
                  dtype="bf16"):
    """Group-mode prefill: the flat problem plus one group query per G consecutive queries."""
    ops = anchor_prefill(T, H, d, K, seed=seed, device=device, dtype="bf16")
    # group queries are built from the unquantised bf16 queries, then prepared like q
    qf = ops["q"].float()
    qbar, wbar = mean_pool_group_queries(qf, ops["w"], G, Hg)
    if dtype == "e4m3":
        kf = ops["k"].float()
        ops.update(as_operands(qf, kf, "e4m3"))
        qbc, qbs = quantize_e4m3_rows(qbar)
        ops.update(qbar=qbc, qbar_scale=qbs)
    else:
        ops.update(qbar=qbar.to(torch.bfloat16).contiguous(), qbar_scale=None)
    ops.update(wbar=wbar, G=G, B=B, Hg=Hg, dtype=dtype)
    return ops


def decode_problem(Bs=32, S=131072, H=64, d=128, K=2048, Hg=16, steps=1, seed=3,
                   device="cpu", k_dtype="e4m3"):
    """Decode: Bs sequences, one bf16 query per sequence per step, each sequence with its
    own key cache.

    At step r (0 <= r < steps) sequence b holds S + r keys and its query sits at position
    S + r - 1; the cache is allocated for S_cap = S + steps - 1 keys. Query anchors drift
    one at a time every 16 steps. Returns the cache as e4m3 codes + per-key fp32 scales (or
    bf16), the per-step queries q_steps [steps, Bs, H, d] bf16 and gates w_steps
    [steps, Bs, H], and the group query of each step (its first Hg heads and their gates),
    which bank refreshes use.
    """
    S_cap = S + steps - 1
    caches, qs, ws = [], [], []
    for b in range(Bs):
        st = AnchorStructure(d, seed * 1000 + b, device, block=16)
        caches.append(st.keys(S_cap))
        qs.append(st.queries(steps, H, pos0=S - 1))
        ws.append(st.gates(steps, H))
    kf = torch.stack(caches)                                   # [Bs, S_cap, d]
    q_steps = torch.stack(qs, dim=1).to(torch.bfloat16).contiguous()   # [steps, Bs, H, d]
    w_steps = torch.stack(ws, dim=1).contiguous()               # [steps, Bs, H]
    if k_dtype == "e4m3":
        kc, ks = quantize_e4m3_rows(kf.reshape(Bs * S_cap, d))
        k, k_scale = kc.reshape(Bs, S_cap, d), ks.reshape(Bs, S_cap)
    else:
        k, k_scale = kf.to(torch.bfloat16).contiguous(), None
    return dict(q_steps=q_steps, w_steps=w_steps, k=k, k_scale=k_scale,
                Bs=Bs, S=S, S_cap=S_cap, steps=steps, H=H, d=d, K=K, Hg=Hg,
                q_dtype="bf16", k_dtype=k_dtype)


def decode_seq_len(prob, step):
    """Keys visible to each sequence at decode step ``step`` (int32 [Bs])."""
    return torch.full((prob["Bs"],), prob["S"] + step, dtype=torch.int32,
                      device=prob["k"].device)


def group_indexer_problem(T, d_c=1536, d_h=7168, H_S=16, d=128, seed=4, device="cpu"):
    """Inputs of the trained group indexer (query latents, normalized hidden states) with
    synthetic weights: cq [T, d_c] and h [T, d_h] ~ N(0, 1) (post-normalization activations),
    W_pool [d_c, 3 d_c], W_Q [H_S d, d_c] and W_G [H_S, d_h] ~ N(0, 1 / fan-in), all bf16."""
    gen = _gen(seed, device)
    bf = torch.bfloat16
    return dict(
        cq=_randn(gen, (T, d_c), device).to(bf),
        h=_randn(gen, (T, d_h), device).to(bf),
        w_pool=_randn(gen, (d_c, 3 * d_c), device, 1.0 / math.sqrt(3 * d_c)).to(bf),
        w_q=_randn(gen, (H_S * d, d_c), device, 1.0 / math.sqrt(d_c)).to(bf),
        w_g=_randn(gen, (H_S, d_h), device, 1.0 / math.sqrt(d_h)).to(bf),
        H_S=H_S, d=d)
