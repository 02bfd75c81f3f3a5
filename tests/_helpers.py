"""Shared pieces of the GPU parity tests: oracle-side expected values (oracle/
and synth only) and the FFN tolerance check."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import ffn as of
from oracle import layout as ol
from oracle import quantize as oq

# FFN tolerance for bf16 activations with fp32 accumulation (stated for the
# method's routed expert FFN): relative Frobenius error and max abs error
# relative to the oracle's largest magnitude.
REL_FRO = 5e-3
MAX_ABS_REL = 2e-2


def check_ffn(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got))
    nref = np.linalg.norm(ref)
    if nref == 0.0:
        assert np.all(got == 0.0)
        return 0.0, 0.0
    rel = np.linalg.norm(got - ref) / nref
    mx = np.abs(got - ref).max() / np.abs(ref).max()
    assert rel <= REL_FRO, f"rel Frobenius {rel:.3e} > {REL_FRO}"
    assert mx <= MAX_ABS_REL, f"max abs {mx:.3e} > {MAX_ABS_REL} * max|ref|"
    return rel, mx


class OracleExpert:
    """Oracle view of one expert: absmax, scale, codes, packed stream, dequantized mats."""

    def __init__(self, master_fp16: np.ndarray, H: int, F: int, b: int):
        self.H, self.F, self.b = H, F, b
        self.m, self.s, self.k = oq.quantize_expert(master_fp16, b)

    def stream(self) -> np.ndarray:
        H, F, b = self.H, self.F, self.b
        u = oq.offset_codes(self.k, b)
        return ol.expert_stream(u[:F * H].reshape(F, H), u[F * H:2 * F * H].reshape(F, H),
                                u[2 * F * H:].reshape(H, F), b).reshape(-1)

    def mats(self):
        H, F = self.H, self.F
        d = oq.dequantize(self.k, self.s)
        return (d[:F * H].reshape(F, H), d[F * H:2 * F * H].reshape(F, H),
                d[2 * F * H:].reshape(H, F))


def workload_masters_cpu(wl, e) -> np.ndarray:
    return synth.expert_weights(wl, e).numpy()


def workload_masters_gpu(wl, device="cuda"):
    out = []
    for e in range(wl.E):
        t = torch.empty(wl.W_e, dtype=torch.float16, device=device)
        synth.fill_expert_weights(wl, e, t)
        out.append(t)
    return out


def oracle_moe(x_bf16: torch.Tensor, ids: np.ndarray, w: np.ndarray, mats_of, E: int,
               tokens=None) -> np.ndarray:
    return of.moe_ffn(x_bf16.double().cpu().numpy(), ids, w, mats_of, E, tokens=tokens)
