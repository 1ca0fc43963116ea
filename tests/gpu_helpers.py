"""Shared helpers of the GPU parity tests: host->device transfer of generator
output and the tolerance checks of the hot path.

Tolerances (written out here and nowhere else):
  attention bf16 inputs, fp32 accumulation:  max-abs 2e-2, mean-abs 2e-3 over
      every compared output element; lse abs 2e-2.  The bar is the one the
      method's target states for bf16; lse has no stated bar — its error comes
      from the bf16 rounding of the rotated query (relative 2^-9 per element,
      about 1e-3 on a unit-variance score) plus the bf16 probabilities of the
      P.V product, so 2e-2 leaves an order of magnitude of margin.
  attention fp32 inputs:  max-abs 1e-4, mean-abs 1e-5, lse 1e-4 (fp32
      accumulation over <= 4200 keys, relative rounding ~1e-6).
  readout log-probs: abs 5e-3 (bf16) / 1e-4 (fp32); choices bit-exact except
      where the oracle's top-two log-prob gap is under 1e-3.
"""
import numpy as np
import torch

import synth

TOL = {
    synth.BF16: dict(max_abs=2e-2, mean_abs=2e-3, lse=2e-2, logprob=5e-3),
    synth.F32: dict(max_abs=1e-4, mean_abs=1e-5, lse=1e-4, logprob=1e-4),
}
NEAR_TIE = 1e-3


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_attn(out_gpu: np.ndarray, lse_gpu: np.ndarray, out_ref: np.ndarray, lse_ref: np.ndarray, dtype: str,
               what: str = ""):
    tol = TOL[dtype]
    err = np.abs(out_gpu - out_ref)
    assert np.all(np.isfinite(out_gpu)), f"{what}: non-finite outputs"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= tol["max_abs"], f"{what}: max-abs {mx:.3g} > {tol['max_abs']}"
    assert mean <= tol["mean_abs"], f"{what}: mean-abs {mean:.3g} > {tol['mean_abs']}"
    if lse_gpu is not None:
        le = float(np.abs(lse_gpu - lse_ref).max())
        assert le <= tol["lse"], f"{what}: lse max-abs {le:.3g} > {tol['lse']}"
    return mx, mean


def check_readout(lp_gpu, ch_gpu, ref, dtype: str, what: str = ""):
    tol = TOL[dtype]["logprob"]
    ok = np.isfinite(ref["logprob"])
    assert np.array_equal(np.isfinite(lp_gpu), ok), f"{what}: NaN pattern differs"
    if ok.any():
        e = float(np.abs(lp_gpu[ok] - ref["logprob"][ok]).max())
        assert e <= tol, f"{what}: logprob max-abs {e:.3g} > {tol}"
    decided = ~(ref["gap"] < NEAR_TIE)
    mism = np.nonzero((ch_gpu != ref["choice"]) & decided)[0]
    assert mism.size == 0, f"{what}: choice mismatch in sets {mism[:10]} (gpu {ch_gpu[mism[:10]]}, ref {ref['choice'][mism[:10]]})"


def compact_lm_head(cfg, toks: np.ndarray):
    """Only the option rows of the LM head are ever read by the readout, so a
    [V, H] device matrix that holds exactly those rows (zeros elsewhere) gives
    the same results as the full one; the oracle gets the same rows compacted
    with remapped token ids.  Returns (device W, oracle W, remapped tokens)."""
    uniq, inv = np.unique(toks, return_inverse=True)
    rows = synth.lm_head_rows(cfg.seed, cfg.V, cfg.H, uniq, cfg.dtype, cfg.w_std)
    Wd = torch.zeros((cfg.V, cfg.H), dtype=torch.bfloat16 if cfg.dtype == synth.BF16 else torch.float32,
                     device="cuda")
    Wd[torch.from_numpy(uniq).long().cuda()] = dev(rows)
    return Wd, rows, inv.astype(np.int32)
