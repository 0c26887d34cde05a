"""Workload tensors for the parity tests, built twice and independently:

* :class:`DeviceLayer` -- drawn on the GPU by ``synth`` and quantised by the
  library under test (``jmoe_quantize``);
* :class:`OracleLayer` -- drawn on the host by ``synth`` and quantised by the
  CPU oracle, one expert at a time and only for the experts a check needs.

Nothing computed by the CUDA path ever becomes an oracle input.
"""
from __future__ import annotations

import numpy as np

import oracle
import synth
from synth.workloads import SIGMA_R, SIGMA_W, SIGMA_X, Workload

MAX_ABS_REL = 2e-2   # max |out - ref| <= 2e-2 * max |ref|
MEAN_REL = 5e-3      # sum |out - ref| / sum |ref| <= 5e-3


class DeviceLayer:
    def __init__(self, wl: Workload, T: int | None = None, device: str = "cuda"):
        import torch

        import int8_weight_moe_b200 as jm

        self.wl = wl
        self.T = wl.T if T is None else T
        s, E, d, f = wl.seed, wl.E, wl.d_model, wl.d_ff
        self.x = synth.normal_bf16_gpu(s, synth.X, SIGMA_X, (self.T, d), device=device)
        self.w_router = None
        if not wl.dense:
            self.w_router = synth.normal_f32_gpu(s, synth.WR, SIGMA_R, (E, d), device=device)
        self.bias = None
        if wl.bias is not None:
            self.bias = torch.tensor(wl.bias, dtype=torch.float32, device=device)
        wgu = synth.normal_bf16_gpu(s, synth.WGU, SIGMA_W, (E, 2 * f, d), device=device)
        self.w_gu, self.s_gu = jm.jmoe_quantize(wgu)
        del wgu
        wdn = synth.normal_bf16_gpu(s, synth.WD, SIGMA_W, (E, d, f), device=device)
        self.w_d, self.s_d = jm.jmoe_quantize(wdn)
        del wdn

    def desc(self, path=0, top_k=None):
        import int8_weight_moe_b200 as jm

        return jm.make_desc(self.w_gu, self.s_gu, self.w_d, self.s_d,
                            top_k=self.wl.top_k if top_k is None else top_k, path=path)


class OracleLayer:
    def __init__(self, wl: Workload, T: int | None = None):
        self.wl = wl
        self.T = wl.T if T is None else T
        s, E, d = wl.seed, wl.E, wl.d_model
        self.x_bits = synth.normal_bf16_bits(s, synth.X, SIGMA_X, (self.T, d))
        self.w_router = None if wl.dense else synth.normal_f32(s, synth.WR, SIGMA_R, (E, d))
        self.bias = None if wl.bias is None else np.array(wl.bias, dtype=np.float32)
        self._experts = {}

    def gate_up_rows(self, e: int, r0: int, n: int):
        d, f = self.wl.d_model, self.wl.d_ff
        return synth.normal_bf16_bits(self.wl.seed, synth.WGU, SIGMA_W, (n, d),
                                      start=(e * 2 * f + r0) * d)

    def down_rows(self, e: int, r0: int, n: int):
        d, f = self.wl.d_model, self.wl.d_ff
        return synth.normal_bf16_bits(self.wl.seed, synth.WD, SIGMA_W, (n, f),
                                      start=(e * d + r0) * f)

    def expert(self, e: int):
        if e not in self._experts:
            d, f = self.wl.d_model, self.wl.d_ff
            qg, sg = oracle.quantize(self.gate_up_rows(e, 0, 2 * f))
            qd, sd = oracle.quantize(self.down_rows(e, 0, d))
            self._experts[e] = (qg, sg, qd, sd)
        return self._experts[e]

    def route(self):
        return oracle.route(self.x_bits, self.w_router, self.wl.top_k, self.bias)

    def forward_tokens(self, tokens, ids, gates):
        """fp64 layer output for the rows ``tokens`` with the given routing."""
        tokens = np.asarray(tokens)
        ids_t = np.asarray(ids)[tokens]
        need = sorted(set(int(e) for e in ids_t.reshape(-1)))
        E = self.wl.E
        tables = [[None] * E for _ in range(4)]
        for e in need:
            for i, a in enumerate(self.expert(e)):
                tables[i][e] = a
        return oracle.moe_forward(self.x_bits[tokens], ids_t, np.asarray(gates)[tokens],
                                  *tables)

    def dense_forward_tokens(self, tokens):
        qg, sg, qd, sd = self.expert(0)
        return oracle.mlp_forward(self.x_bits[np.asarray(tokens)], qg, sg, qd, sd)


def gate_sum_bound(top_k: int) -> float:
    """Largest |sum_j g_j - 1| the device's fp32 renormalisation can give:
    the selected probabilities are summed in fp32 in selection order (top_k - 1
    roundings of relative size <= 2^-24) and each gate is one correctly
    rounded fp32 division (relative error <= 2^-24), so the sum is within
    top_k * 2^-24 of 1, up to second-order terms (the 2^-20 slack)."""
    return top_k * 2.0 ** -24 * (1.0 + 2.0 ** -20)


def boundary_tokens(ids, E: int, top_k: int, tile: int = 128, experts=None):
    """Tokens whose assignments sit where the expert kernels' tiling changes.

    The assignments are grouped by expert with the oracle's stable counting
    sort (the method's dispatch).  For every expert: its first and last
    grouped row; for the experts in ``experts`` (all when None): both rows
    on either side of every multiple of ``tile`` (the tensor-core path's
    128-row MMA halves, 256-row tiles and raster groups all start at such
    multiples).  Returns the sorted tokens of those rows."""
    ids = np.asarray(ids, dtype=np.int32)
    offsets, perm, _ = oracle.permute(ids, E)
    rows = set()
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        rows.update((lo, hi - 1))
        if experts is None or e in experts:
            for b in range(tile, hi - lo, tile):
                rows.update((lo + b - 1, lo + b))
    return sorted(set(int(perm[r]) // top_k for r in rows))


def assert_close(got, ref, what=""):
    """The parity bar for floating-point outputs (bf16 I/O, fp32 accumulation)."""
    rep = oracle.tolerance_report(got, ref)
    assert rep["max_rel"] <= MAX_ABS_REL and rep["mean_rel"] <= MEAN_REL, (what, rep)
    return rep


def bf16_to_f64(t):
    import torch

    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)
