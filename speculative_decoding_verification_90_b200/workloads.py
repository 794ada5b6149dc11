"""Seeded synthetic inputs for the verification step.

This module only draws random numbers and lays them out; it holds none of the
verification arithmetic (no softmax, no acceptance test, no CDF).  Both the
CUDA path and the CPU oracle are fed from it, in tests and in the benchmark.

Draft tokens are drawn from the draft distribution softmax(draft_logits / T)
with the Gumbel-max construction (argmax of logits / T plus Gumbel noise),
which samples that distribution exactly without normalising it.

Logits are returned as float32, or for bf16 workloads as uint16 arrays that
hold bf16 bit patterns (round-to-nearest-even of the float32 draws).

Workloads (sizes as in the benchmark configurations the project is measured
on; no public dataset stands behind any of them):

* ``char_level``   B=1 per call, gamma=4, V=256, fp32, T=1; target N(0, 3^2),
                   draft = 0.8 target + 0.2 fresh N(0, 3^2); ``calls``
                   independent calls stacked along the batch axis.
* ``exactness``    B=60000 rows sharing one position, gamma=1, V=4096, fp32;
                   one fixed target row pair N(0, 3^2) and one fixed draft row
                   (1-beta) z + beta w, w ~ N(0, 3^2); beta is chosen offline
                   so that TV(p, q) is the pages' 0.657; fresh tokens and
                   uniforms per row.
* ``b8_g3_v32000`` B=8, gamma=3, V=32000, bf16, T=0.7; target N(0, 2.5^2),
                   draft = 0.9 target + 0.1 N(0, 2.5^2).
* ``b64_g8_v128256`` B=64, gamma=8, V=128256, bf16, T=1; target N(0, 3^2)
                   plus +8 on one uniformly chosen token per row; draft =
                   0.85 target + 0.15 N(0, 3^2).
* ``multibranch``  32 sequences x 8 branches = 256 rows, gamma=5, V=152064,
                   bf16, T=1.  Per sequence a branch point bp ~ U{1..gamma}:
                   target rows, draft rows and draft tokens at positions
                   j < bp are shared by the sequence's branches; positions
                   j >= bp are fresh N(0, 3^2) draws per branch.  Draft =
                   0.8 target + 0.2 N(0, 3^2).  Also given as distinct rows
                   plus row maps, for the shared-row entry point.
* ``lmhead``       fused-step inputs: 64 sequences, gamma=8, V=128256,
                   hidden 4096, bf16 hidden states and output layer whose
                   logits are N(0, 3^2) (see the function).
* ``gate_tree``    fold-gate inputs: 128 sequences x 8 candidate branches, one
                   block of 32 positions, hidden size 4096, bf16; a random
                   tree per sequence and a perturbation that peaks at each
                   child's newly revealed position (see the function).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

F32 = "f32"
BF16 = "bf16"
MAPPED_KEYS = ("target_rows", "target_map", "draft_rows", "draft_map")


@dataclass
class Workload:
    name: str
    batch: int
    gamma: int
    vocab: int
    dtype: str              # "f32" or "bf16"
    temperature: float
    target: np.ndarray      # [B, gamma+1, V] float32 or uint16 (bf16 bits)
    draft: np.ndarray       # [B, gamma, V]
    tokens: np.ndarray      # int32 [B, gamma]
    u_accept: np.ndarray    # float32 [B, gamma]
    u_resample: np.ndarray  # float32 [B]
    meta: dict = field(default_factory=dict)

    @property
    def elem_size(self) -> int:
        return 4 if self.dtype == F32 else 2

    @property
    def logit_bytes(self) -> int:
        """Bytes of logits the step must read at least once."""
        return self.batch * (2 * self.gamma + 1) * self.vocab * self.elem_size

    def slice(self, lo: int, hi: int) -> "Workload":
        # the distinct-row tables index the whole batch: a slice keeps only the
        # per-position arrays
        meta = {k: v for k, v in self.meta.items() if k not in MAPPED_KEYS}
        return Workload(self.name, hi - lo, self.gamma, self.vocab, self.dtype, self.temperature,
                        self.target[lo:hi], self.draft[lo:hi], self.tokens[lo:hi],
                        self.u_accept[lo:hi], self.u_resample[lo:hi], meta)

    @property
    def mapped(self) -> bool:
        """True if ``meta`` holds distinct rows and row maps (shared-row layout)."""
        return all(k in self.meta for k in MAPPED_KEYS)

    @property
    def unique_logit_bytes(self) -> int:
        """Bytes of the distinct logit rows (the shared-row step reads each once)."""
        if not self.mapped:
            return self.logit_bytes
        rows = self.meta["target_rows"].shape[0] + self.meta["draft_rows"].shape[0]
        return rows * self.vocab * self.elem_size


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (NaN kept quiet)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    nan = np.isnan(x)
    out = rounded.astype(np.uint16)
    if nan.any():
        out[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return out


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> the float32 values they denote (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _normal(rng: np.random.Generator, shape, sigma: float) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32) * np.float32(sigma)


def gumbel_max_tokens(rng: np.random.Generator, logits: np.ndarray, temperature: float,
                      block_rows: int = 64) -> np.ndarray:
    """One draw per row from softmax(logits / T) by the Gumbel-max construction.

    ``logits`` is float32 [..., V] (the values the verifier will see).
    """
    flat = logits.reshape(-1, logits.shape[-1])
    out = np.empty(flat.shape[0], np.int32)
    tiny = np.float32(np.finfo(np.float32).tiny)
    inv_t = np.float32(1.0 / temperature)
    for r0 in range(0, flat.shape[0], block_rows):
        blk = flat[r0:r0 + block_rows]
        u = rng.random(blk.shape, dtype=np.float32)
        np.maximum(u, tiny, out=u)
        g = -np.log(-np.log(u))
        g += blk * inv_t
        out[r0:r0 + block_rows] = np.argmax(g, axis=1)
    return out.reshape(logits.shape[:-1])


def _finish(name, dtype, T, target_f32, draft_f32, rng, meta=None, tokens=None) -> Workload:
    """Round to the storage dtype, draw tokens from the stored draft logits, draw uniforms."""
    if dtype == BF16:
        tgt = bf16_bits(target_f32)
        drf = bf16_bits(draft_f32)
        drf_seen = bits_to_f32(drf)
    else:
        tgt = np.ascontiguousarray(target_f32, dtype=np.float32)
        drf = np.ascontiguousarray(draft_f32, dtype=np.float32)
        drf_seen = drf
    B, G, V = drf.shape
    if tokens is None:
        tokens = gumbel_max_tokens(rng, drf_seen, T) if G > 0 else np.zeros((B, 0), np.int32)
    u_acc = rng.random((B, G), dtype=np.float32)
    u_res = rng.random(B, dtype=np.float32)
    return Workload(name, B, G, V, dtype, float(T), tgt, drf, tokens.astype(np.int32),
                    u_acc, u_res, meta or {})


def char_level(calls: int = 1000, seed: int = 0) -> Workload:
    """B=1 per call, gamma=4, V=256, fp32, T=1; ``calls`` calls stacked on the batch axis."""
    rng = np.random.default_rng(seed)
    G, V = 4, 256
    tgt = _normal(rng, (calls, G + 1, V), 3.0)
    drf = np.float32(0.8) * tgt[:, :G] + np.float32(0.2) * _normal(rng, (calls, G, V), 3.0)
    return _finish("char_level_b1_g4_v256_f32", F32, 1.0, tgt, drf, rng, {"calls": calls})


def exactness_rows(seed: int = 0, vocab: int = 4096):
    """The fixed target row pair z (position 0 and the bonus position) and the fixed noise w."""
    rng = np.random.default_rng(seed)
    z = _normal(rng, (2, vocab), 3.0)
    w = _normal(rng, (vocab,), 3.0)
    return z, w


def exactness_draft_row(z: np.ndarray, w: np.ndarray, beta: float) -> np.ndarray:
    return ((1.0 - beta) * z[0].astype(np.float64) + beta * w.astype(np.float64)).astype(np.float32)


def exactness(beta: float, batch: int = 60000, seed: int = 0, vocab: int = 4096) -> Workload:
    """B rows sharing one position (gamma=1, V=4096, fp32, T=1), fresh tokens/uniforms per row."""
    z, w = exactness_rows(seed, vocab)
    d = exactness_draft_row(z, w, beta)
    rng = np.random.default_rng(seed + 1)
    tgt = np.broadcast_to(z[None], (batch, 2, vocab))
    drf = np.broadcast_to(d[None, None], (batch, 1, vocab))
    tokens = gumbel_max_tokens(rng, np.ascontiguousarray(drf), 1.0, block_rows=2048)
    return _finish("exactness_b60000_g1_v4096_f32", F32, 1.0, np.ascontiguousarray(tgt),
                   np.ascontiguousarray(drf), rng, {"beta": beta}, tokens=tokens)


def b8_g3_v32000(seed: int = 0) -> Workload:
    rng = np.random.default_rng(seed)
    B, G, V = 8, 3, 32000
    tgt = _normal(rng, (B, G + 1, V), 2.5)
    drf = np.float32(0.9) * tgt[:, :G] + np.float32(0.1) * _normal(rng, (B, G, V), 2.5)
    return _finish("b8_g3_v32000_bf16", BF16, 0.7, tgt, drf, rng)


def b64_g8_v128256(seed: int = 0, batch: int = 64) -> Workload:
    rng = np.random.default_rng(seed)
    B, G, V = batch, 8, 128256
    tgt = _normal(rng, (B, G + 1, V), 3.0)
    peak = rng.integers(0, V, size=(B, G + 1))
    np.add.at(tgt, (np.arange(B)[:, None], np.arange(G + 1)[None, :], peak), np.float32(8.0))
    drf = np.float32(0.85) * tgt[:, :G] + np.float32(0.15) * _normal(rng, (B, G, V), 3.0)
    return _finish("b64_g8_v128256_bf16", BF16, 1.0, tgt, drf, rng)


def multibranch(seed: int = 0, sequences: int = 32, branches: int = 8, gamma: int = 5,
                vocab: int = 152064) -> Workload:
    """sequences x branches rows sharing target/draft rows and tokens before a branch point.

    Besides the per-position arrays, ``meta`` holds each distinct row once:
    ``target_rows`` / ``draft_rows`` (bf16 bits) and ``target_map`` [B, G+1] /
    ``draft_map`` [B, G] (int32), with ``target[b, j] == target_rows[target_map[b, j]]``.
    """
    rng = np.random.default_rng(seed)
    S, K, G, V = sequences, branches, gamma, vocab
    B = S * K
    points = rng.integers(1, G + 1, size=S) if G > 0 else np.zeros(S, np.int64)
    t_parts, d_parts = [], []
    t_map = np.empty((B, G + 1), np.int32)
    d_map = np.empty((B, G), np.int32)
    shared = np.zeros((B, G), bool)
    nt = nd = 0
    for s in range(S):
        bp = int(points[s])
        base_t = _normal(rng, (bp, V), 3.0)
        base_d = np.float32(0.8) * base_t + np.float32(0.2) * _normal(rng, (bp, V), 3.0)
        t_parts.append(base_t)
        d_parts.append(base_d)
        t0, d0 = nt, nd
        nt += bp
        nd += bp
        for k in range(K):
            b = s * K + k
            t_map[b, :bp] = t0 + np.arange(bp)
            d_map[b, :bp] = d0 + np.arange(bp)
            own_t = _normal(rng, (G + 1 - bp, V), 3.0)
            t_parts.append(own_t)
            t_map[b, bp:] = nt + np.arange(G + 1 - bp)
            nt += G + 1 - bp
            if bp < G:
                d_parts.append(np.float32(0.8) * own_t[:G - bp]
                               + np.float32(0.2) * _normal(rng, (G - bp, V), 3.0))
                d_map[b, bp:] = nd + np.arange(G - bp)
                nd += G - bp
            shared[b, :bp] = True
    t_rows = bf16_bits(np.concatenate(t_parts))
    del t_parts
    d_rows = bf16_bits(np.concatenate(d_parts)) if d_parts else np.zeros((0, V), np.uint16)
    del d_parts
    # tokens: one draw per (sequence, shared position), one per (row, private position)
    seen = bits_to_f32(d_rows)
    tokens = np.empty((B, G), np.int32)
    for s in range(S):
        bp = int(points[s])
        rows = slice(s * K, (s + 1) * K)
        if bp > 0:
            tokens[rows, :bp] = gumbel_max_tokens(rng, seen[d_map[s * K, :bp]][None], 1.0)[0][None]
        if bp < G:
            tokens[rows, bp:] = gumbel_max_tokens(rng, seen[d_map[rows, bp:]], 1.0)
    del seen
    u_acc = rng.random((B, G), dtype=np.float32)
    u_res = rng.random(B, dtype=np.float32)
    return Workload("multibranch_32x8_g5_v152064_bf16", B, G, V, BF16, 1.0, t_rows[t_map],
                    d_rows[d_map], tokens, u_acc, u_res,
                    {"sequences": S, "branches": K, "branch_points": points.tolist(),
                     "shared": shared, "target_rows": t_rows, "target_map": t_map,
                     "draft_rows": d_rows, "draft_map": d_map})


def random_maps(seed: int = 0, batch: int = 24, gamma: int = 4, vocab: int = 5000,
                target_rows: int = 40, draft_rows: int = 30, dtype: str = F32,
                temperature: float = 1.0) -> Workload:
    """Distinct rows with arbitrary many-to-one row maps (positions of different
    sequences, and a target and a bonus position, may share a row).

    Target rows N(0, 3^2); each draft row is 0.8 x a random target row + 0.2
    N(0, 3^2).  Maps are uniform over the rows, then the first rows are pinned
    so that every row is used at least once.  Tokens are drawn from the
    materialised draft rows.
    """
    rng = np.random.default_rng(seed)
    B, G, V = batch, gamma, vocab
    if not 1 <= target_rows <= B * (G + 1) or (G > 0 and not 1 <= draft_rows <= B * G):
        raise ValueError("row counts must be within [1, positions]")
    t_f = _normal(rng, (target_rows, V), 3.0)
    d_rows_n = draft_rows if G > 0 else 0
    src = rng.integers(0, target_rows, size=d_rows_n)
    d_f = np.float32(0.8) * t_f[src] + np.float32(0.2) * _normal(rng, (d_rows_n, V), 3.0)
    t_map = rng.integers(0, target_rows, size=(B, G + 1)).astype(np.int32)
    t_map.reshape(-1)[rng.permutation(B * (G + 1))[:target_rows]] = np.arange(target_rows)
    d_map = rng.integers(0, max(d_rows_n, 1), size=(B, G)).astype(np.int32)
    if G > 0:
        d_map.reshape(-1)[rng.permutation(B * G)[:d_rows_n]] = np.arange(d_rows_n)
    if dtype == BF16:
        t_st, d_st = bf16_bits(t_f), bf16_bits(d_f)
        d_seen = bits_to_f32(d_st)
    else:
        t_st, d_st, d_seen = t_f, d_f, d_f
    tokens = (gumbel_max_tokens(rng, d_seen[d_map], temperature) if G > 0
              else np.zeros((B, 0), np.int32))
    u_acc = rng.random((B, G), dtype=np.float32)
    u_res = rng.random(B, dtype=np.float32)
    return Workload(f"random_maps_b{B}_g{G}_v{V}_{dtype}", B, G, V, dtype, float(temperature),
                    t_st[t_map], d_st[d_map], tokens.astype(np.int32), u_acc, u_res,
                    {"target_rows": t_st, "target_map": t_map, "draft_rows": d_st,
                     "draft_map": d_map})


@dataclass
class GateWorkload:
    """Hidden states of candidate branches at one layer input, and their tree."""
    name: str
    branches: int
    positions: int
    dim: int
    dtype: str              # "f32" or "bf16"
    tau: float
    hidden: np.ndarray      # [branches, positions, dim] float32 or uint16 (bf16 bits)
    parent: np.ndarray      # int32 [branches], -1 for a branch without a parent
    meta: dict = field(default_factory=dict)

    @property
    def elem_size(self) -> int:
        return 4 if self.dtype == F32 else 2

    @property
    def rows(self) -> int:
        return self.branches * self.positions

    def rows_read(self) -> int:
        """Rows the gate must read at least once: every row of a branch that has a
        parent (as the child) or that is some branch's parent."""
        nb = self.branches
        p = self.parent
        has_parent = (p >= 0) & (p < nb)
        is_parent = np.zeros(nb, bool)
        is_parent[p[has_parent]] = True
        return int((has_parent | is_parent).sum()) * self.positions


def gate_tree(seed: int = 0, sequences: int = 128, branches: int = 8, positions: int = 32,
              dim: int = 4096, dtype: str = BF16, tau: float = 0.05, amplitude: float = 0.5,
              width: float = 2.0, floor: float = 0.01) -> GateWorkload:
    """Per sequence a tree of ``branches`` candidates over one block of ``positions``.

    Branch 0 of a sequence has no parent and holds N(0, 1) hidden states; branch
    k >= 1 takes a parent uniformly among branches 0..k-1 of its sequence and a
    revealed position r ~ U{0..positions-1}, and its hidden state at position j
    is the parent's plus N(0, 1) noise scaled by
    amplitude * exp(-|j - r| / width) + floor, so the difference is largest at
    the newly revealed position and ripples out to its neighbours.  States are
    stored in ``dtype`` (bf16: round to nearest even); a child is built from its
    parent's stored values.
    """
    rng = np.random.default_rng(seed)
    nb = sequences * branches
    parent = np.empty(nb, np.int32)
    revealed = np.full(nb, -1, np.int64)
    store = bf16_bits if dtype == BF16 else (lambda a: np.ascontiguousarray(a, np.float32))
    seen = bits_to_f32 if dtype == BF16 else (lambda a: a)
    hidden = np.empty((nb, positions, dim), np.uint16 if dtype == BF16 else np.float32)
    j = np.arange(positions, dtype=np.float32)[:, None]
    for s in range(sequences):
        b0 = s * branches
        parent[b0] = -1
        hidden[b0] = store(rng.standard_normal((positions, dim), dtype=np.float32))
        for k in range(1, branches):
            c = b0 + k
            p = b0 + int(rng.integers(0, k))
            r = int(rng.integers(0, positions))
            parent[c] = p
            revealed[c] = r
            scale = (np.float32(amplitude) * np.exp(-np.abs(j - np.float32(r)) / np.float32(width))
                     + np.float32(floor)).astype(np.float32)
            noise = rng.standard_normal((positions, dim), dtype=np.float32)
            hidden[c] = store(seen(hidden[p]) + scale * noise)
    name = f"gate_{sequences}x{branches}_p{positions}_d{dim}_{dtype}"
    return GateWorkload(name, nb, positions, dim, dtype, float(tau), hidden, parent,
                        {"sequences": sequences, "branches_per_sequence": branches,
                         "revealed": revealed})


@dataclass
class LmWorkload:
    """Hidden states and output-layer weights (bf16 bits) for the fused step."""
    name: str
    batch: int
    gamma: int
    vocab: int
    hidden: int
    temperature: float
    target_hidden: np.ndarray   # uint16 [B, gamma+1, hidden]
    target_weight: np.ndarray   # uint16 [vocab, hidden]
    draft_hidden: np.ndarray    # uint16 [B, gamma, hidden]
    draft_weight: np.ndarray    # uint16 [vocab, hidden] (the target's when shared)
    tokens: np.ndarray          # int32 [B, gamma]
    u_accept: np.ndarray        # float32 [B, gamma]
    u_resample: np.ndarray      # float32 [B]
    meta: dict = field(default_factory=dict)


def lmhead(seed: int = 0, batch: int = 64, gamma: int = 8, vocab: int = 128256,
           hidden: int = 4096, shared_weight: bool = True, temperature: float = 1.0) -> LmWorkload:
    """Output-layer inputs with logits distributed like the b64_g8_v128256 batch.

    Target hidden states N(0, 1); weights N(0, (3/sqrt(hidden))^2), so a logit
    is N(0, 3^2); draft hidden states 0.9 x the target's at the same position +
    0.1 x N(0, 1); the draft uses the target's output layer (shared) or
    0.85 x it + 0.15 x fresh noise.  All stored as bf16.  Draft tokens are drawn
    from softmax(draft logits / T) by Gumbel-max on float32 logits of the stored
    values (computed here in row blocks).
    """
    rng = np.random.default_rng(seed)
    B, G, V, D = batch, gamma, vocab, hidden
    ht = bf16_bits(rng.standard_normal((B, G + 1, D), dtype=np.float32))
    w = np.empty((V, D), np.uint16)
    sigma = np.float32(3.0 / np.sqrt(D))
    for v0 in range(0, V, 8192):
        w[v0:v0 + 8192] = bf16_bits(rng.standard_normal((min(8192, V - v0), D), dtype=np.float32)
                                    * sigma)
    hd = bf16_bits(np.float32(0.9) * bits_to_f32(ht[:, :G])
                   + np.float32(0.1) * rng.standard_normal((B, G, D), dtype=np.float32))
    if shared_weight:
        wd = w
    else:
        wd = np.empty_like(w)
        for v0 in range(0, V, 8192):
            n = min(8192, V - v0)
            wd[v0:v0 + n] = bf16_bits(np.float32(0.85) * bits_to_f32(w[v0:v0 + n])
                                      + np.float32(0.15) * sigma
                                      * rng.standard_normal((n, D), dtype=np.float32))
    tokens = np.zeros((B, G), np.int32)
    if G > 0:
        hdf = bits_to_f32(hd).reshape(B * G, D)
        best = np.full(B * G, -np.inf, np.float32)
        arg = np.zeros(B * G, np.int64)
        tiny = np.float32(np.finfo(np.float32).tiny)
        for v0 in range(0, V, 8192):
            n = min(8192, V - v0)
            logits = hdf @ bits_to_f32(wd[v0:v0 + n]).T
            u = rng.random(logits.shape, dtype=np.float32)
            np.maximum(u, tiny, out=u)
            g = logits / np.float32(temperature) - np.log(-np.log(u))
            j = np.argmax(g, axis=1)
            val = g[np.arange(g.shape[0]), j]
            better = val > best
            best[better] = val[better]
            arg[better] = v0 + j[better]
        tokens = arg.astype(np.int32).reshape(B, G)
    u_acc = rng.random((B, G), dtype=np.float32)
    u_res = rng.random(B, dtype=np.float32)
    name = f"lmhead_b{B}_g{G}_v{V}_d{D}_bf16" + ("" if shared_weight else "_two_heads")
    return LmWorkload(name, B, G, V, D, float(temperature), ht, w, hd, wd, tokens, u_acc, u_res,
                      {"shared_weight": shared_weight})


REGISTRY = {
    "char_level": char_level,
    "b8_g3_v32000": b8_g3_v32000,
    "b64_g8_v128256": b64_g8_v128256,
    "multibranch": multibranch,
}
