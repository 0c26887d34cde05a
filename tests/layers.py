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

    def forward_tokens(self, tokens, ids, gates, round_h_bf16=False):
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
                                  *tables, round_h_bf16=round_h_bf16)

    def dense_forward_tokens(self, tokens):
        qg, sg, qd, sd = self.expert(0)
        return oracle.mlp_forward(self.x_bits[np.asarray(tokens)], qg, sg, qd, sd)


def assert_close(got, ref, what=""):
    """The parity bar for floating-point outputs (bf16 I/O, fp32 accumulation)."""
    rep = oracle.tolerance_report(got, ref)
    assert rep["max_rel"] <= MAX_ABS_REL and rep["mean_rel"] <= MEAN_REL, (what, rep)
    return rep


def bf16_to_f64(t):
    import torch

    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)
