"""A host model of the context-parallel phases, for the CPU tests of the exchange logic.

It runs the same phase sequence as libspa's context-parallel kernels and reads and
writes the same exchange-buffer layouts (byte tensors: stats [R][X][n_chunks][G] float
pairs, hist1/hist2 [X][4096] uint64 summed over the ranks, hist3 [R][X][64][2] uint64,
with X = B * n_ret rows, one per retrieval slice, sequence-major; out_all
[R][B][Hq][128] and lse_all [R][B][Hq] float32), in float64 NumPy, so that the
orchestration in ``head_partitioned_sparse_b200.context_parallel`` and the gloo
all-gathers can be tested without a GPU, and so that the phase decomposition itself
(merging per-rank softmax statistics, exact integer histograms summed over ranks, the
tie quota taken rank by rank) is checked against the oracle.  Test code only.
"""
from __future__ import annotations

import math

import numpy as np

import oracle as O

LOG2E = 1.4426950408889634
CHUNK = 4096
BINS1, BINS2, BINS3 = 4096, 4096, 64


def n_chunks(C: int) -> int:
    return -(-C // CHUNK)


def exchange_sizes(B: int, Hq: int, Hkv: int, C: int, R: int, head_mask):
    """Byte sizes of the exchange buffers (the layout spa_cp_exchange_sizes reports):
    statistics and histograms for the retrieval slices only, hist1 and hist2 without a
    slot per rank (summed)."""
    G, X = Hq // Hkv, B * int(sum(1 for v in head_mask if v))
    return (R * X * n_chunks(C) * G * 8, X * BINS1 * 8, X * BINS2 * 8, R * X * BINS3 * 16,
            R * B * Hq * 128 * 4, R * B * Hq * 4)


def mass_q(u: np.ndarray) -> np.ndarray:
    """Probability bit patterns -> exact masses in units of 2^-63 (0 below 2^-40)."""
    u = np.asarray(u, np.uint64)
    e = (u >> np.uint64(23)) & np.uint64(0xFF)
    sig = (u & np.uint64(0x7FFFFF)) | np.uint64(0x800000)
    sh = np.clip(e.astype(np.int64), 87, 127) - 87
    return np.where(e >= 87, sig << sh.astype(np.uint64), np.uint64(0))


def cut_desc(h, above: int, target: int):
    """Bin where above + cumulative mass (bins visited from the highest) reaches target."""
    cum = above
    for d in range(len(h) - 1, -1, -1):
        nx = cum + int(h[d])
        if cum < target <= nx:
            return d, cum
        cum = nx
    return -1, cum


class HostRank:
    """Rank ``rank`` of ``R``: positions [rank C, (rank + 1) C) of every sequence."""

    def __init__(self, inp, idx_bits, rank: int, R: int, C: int, bufs, *, p: float, n_sink: int, window: int):
        self.inp, self.rank, self.R, self.C = inp, rank, R, C
        self.p, self.n_sink, self.window = p, n_sink, window
        self.G = inp.Hq // inp.Hkv
        # exchange row of slice (b, g): b * n_ret + (ordinal of g among the retrieval heads)
        ret = [g for g in range(inp.Hkv) if inp.head_mask[g]]
        self.X = inp.B * len(ret)
        self.xrow = {b * inp.Hkv + g: b * len(ret) + j for b in range(inp.B) for j, g in enumerate(ret)}
        self.nc = n_chunks(C)
        self.pos0 = rank * C
        self.idx = idx_bits
        self.to64 = (lambda a: O.bf16_bits_to_f64(a)) if inp.dtype == "bf16" else (
            lambda a: np.asarray(a, np.float64))
        nb = lambda name: bufs[name].numpy()
        self.stats = nb("stats").view(np.float32).reshape(R, self.X, self.nc, self.G, 2)
        self.h1 = nb("hist1").view(np.uint64).reshape(self.X, BINS1)   # summed over the ranks
        self.h2 = nb("hist2").view(np.uint64).reshape(self.X, BINS2)
        self.h3 = nb("hist3").view(np.uint64).reshape(R, self.X, BINS3, 2)
        self.out_all = nb("out_all").view(np.float32).reshape(R, inp.B, inp.Hq, 128)
        self.lse_all = nb("lse_all").view(np.float32).reshape(R, inp.B, inp.Hq)
        self.bits = {}
        self.cut = {}
        self.rows = {}

    # -- helpers
    def _n(self, b):
        return int(min(max(int(self.inp.seq_lens[b]) - self.pos0, 0), self.C))

    def _slices(self):
        for b in range(self.inp.B):
            for g in range(self.inp.Hkv):
                yield b, g, b * self.inp.Hkv + g

    def _logits(self, b, g):
        inp, G = self.inp, self.G
        hs = range(g * G, (g + 1) * G)
        qi = np.stack([inp.P_q[h].astype(np.float64) @ self.to64(inp.q_pre[b, h]) for h in hs])
        rows = O.bf16_bits_to_f64(self.idx[b, g, self.pos0:self.pos0 + self._n(b)])
        return LOG2E * float(inp.idx_scale) * (rows @ qi.T)      # [n][G]

    # -- phases
    def phase(self, ph: int) -> None:
        getattr(self, ("stats_phase", "mass_phase", "round2", "round3", "attend")[ph])()

    # Each phase clears the summed rows the next phase adds into (as the kernels do), so
    # ranks that share the buffers add into one sum.
    def stats_phase(self):
        self.stats[self.rank] = 0
        self.h1[:] = 0
        for b, g, s in self._slices():
            if not self.inp.head_mask[g]:
                continue
            lg, x = self._logits(b, g), self.xrow[s]
            for c in range(self.nc):
                part = lg[c * CHUNK:(c + 1) * CHUNK]
                if len(part) == 0:
                    self.stats[self.rank, x, c, :, 0] = -np.inf
                    self.stats[self.rank, x, c, :, 1] = 0.0
                    continue
                m = part.max(axis=0)
                self.stats[self.rank, x, c, :, 0] = m
                self.stats[self.rank, x, c, :, 1] = np.exp2(part - m).sum(axis=0)

    def mass_phase(self):
        self.h2[:] = 0
        self.h3[self.rank] = 0
        for b, g, s in self._slices():
            if not self.inp.head_mask[g]:
                continue
            x = self.xrow[s]
            st = self.stats[:, x].reshape(-1, self.G, 2).astype(np.float64)   # all ranks, all chunks
            m, z = st[..., 0], st[..., 1]
            M = m.max(axis=0)
            Z = np.where(np.isfinite(m), z * np.exp2(m - M), 0.0).sum(axis=0)
            pi = (np.exp2(self._logits(b, g) - M) / (self.G * Z)).sum(axis=1).astype(np.float32)
            u = pi.view(np.uint32)
            self.bits[s] = u
            np.add.at(self.h1[x], (u >> 18).astype(np.int64), mass_q(u))

    def round2(self):
        for b, g, s in self._slices():
            if not self.inp.head_mask[g]:
                continue
            x = self.xrow[s]
            total = sum(int(v) for v in self.h1[x])
            target = max(1, math.ceil(float(np.float32(self.p)) * float(total)))
            if self.p >= 1.0 or target > total:
                self.cut[s] = dict(b1=-1)
                continue
            b1, above = cut_desc(self.h1[x], 0, target)
            self.cut[s] = dict(b1=b1, above=above, target=target)
            u = self.bits[s]
            sel = (u >> 18) == b1
            np.add.at(self.h2[x], ((u[sel] >> 6) & 0xFFF).astype(np.int64), mass_q(u[sel]))

    def round3(self):
        for s, cs in self.cut.items():
            if cs["b1"] < 0:
                continue
            x = self.xrow[s]
            b2, above = cut_desc(self.h2[x], cs["above"], cs["target"])
            cs.update(b2=b2, above=above)
            u = self.bits[s]
            sel = (u >> 6) == ((cs["b1"] << 12) | b2)
            d = (u[sel] & 0x3F).astype(np.int64)
            np.add.at(self.h3[self.rank, x, :, 0], d, mass_q(u[sel]))
            np.add.at(self.h3[self.rank, x, :, 1], d, np.uint64(1))

    def attend(self):
        inp = self.inp
        self.out_all[self.rank] = 0
        self.lse_all[self.rank] = -np.inf
        for b, g, s in self._slices():
            L, n = int(inp.seq_lens[b]), self._n(b)
            loc = np.arange(n)
            always = np.isin(self.pos0 + loc, O.sink_window(L, self.n_sink, self.window))
            keep = always.copy()
            if inp.head_mask[g]:
                cs = self.cut[s]
                if cs["b1"] < 0:
                    keep[:] = True
                else:
                    x = self.xrow[s]
                    b3, above = cut_desc(self.h3[:, x, :, 0].sum(axis=0, dtype=np.uint64), cs["above"],
                                         cs["target"])
                    tau = (cs["b1"] << 18) | (cs["b2"] << 6) | b3
                    mt = int(mass_q(np.array([tau], np.uint32))[0])
                    ties = -(-(cs["target"] - above) // mt)
                    before = sum(int(self.h3[r, x, b3, 1]) for r in range(self.rank))
                    quota = min(max(ties - before, 0), int(self.h3[self.rank, x, b3, 1]))
                    u = self.bits[s].astype(np.int64)
                    eq = u == tau
                    keep |= (u > tau) | (eq & (np.cumsum(eq) - 1 < quota))
            rows = loc[keep]
            self.rows[(b, g)] = rows + self.pos0
            if len(rows) == 0:
                continue
            for h in range(g * self.G, (g + 1) * self.G):
                q = O.rope(self.to64(inp.q_pre[b, h]), L - 1, inp.rope_theta)
                K = self.to64(inp.k_cache[b, g, self.pos0 + rows])
                V = self.to64(inp.v_cache[b, g, self.pos0 + rows])
                sc = K @ q / np.sqrt(128.0)
                mx = sc.max()
                w = np.exp(sc - mx)
                self.out_all[self.rank, b, h] = (w @ V) / w.sum()
                self.lse_all[self.rank, b, h] = (mx + np.log(w.sum())) * LOG2E


def combine(out_all: np.ndarray, lse_all: np.ndarray) -> np.ndarray:
    """out = sum_r 2^(lse_r - M) out_r / sum_r 2^(lse_r - M), ranks in order."""
    lse = lse_all.astype(np.float64)
    M = lse.max(axis=0)
    w = np.where(np.isfinite(lse), np.exp2(lse - M), 0.0)
    return (w[..., None] * out_all.astype(np.float64)).sum(axis=0) / w.sum(axis=0)[..., None]
