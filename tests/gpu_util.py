"""Helpers for the GPU tests: host storage arrays <-> torch CUDA tensors, and the
tolerances the attention outputs are held to (max-abs error against the float64
oracle: 1e-4 for float32 caches, 2e-2 for bf16/f16 caches with float32
accumulation)."""

import numpy as np
import torch

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
PA_CODE = {"f32": 0, "bf16": 1, "f16": 2}
ATOL = {"f32": 1e-4, "bf16": 2e-2, "f16": 2e-2}
NAN_BITS = {"f32": np.float32(np.nan), "bf16": np.uint16(0x7FC0), "f16": np.float16(np.nan)}


def to_dev(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if dtype == "bf16":
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(a)
    return t.to(device)


def to_host(t: torch.Tensor, dtype: str) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if dtype == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def out_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().double().cpu().numpy()


def blocks_for(n, bs):
    return (n + bs - 1) // bs


def tables_from_order(lens, bs, order, width):
    """Block tables that give sequence s the next ceil(L_s/bs) blocks of ``order``
    (test setup only; both sides read the same tables)."""
    rows = np.full((len(lens), width), -1, np.int32)
    pos = 0
    for s, L in enumerate(lens):
        n = blocks_for(int(L), bs)
        rows[s, :n] = order[pos:pos + n]
        pos += n
    return rows


def assert_close(got, want, dtype, what=""):
    err = float(np.nanmax(np.abs(got - want))) if got.size else 0.0
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err <= ATOL[dtype], f"{what}: max abs error {err:.3g} > {ATOL[dtype]}"
    return err
