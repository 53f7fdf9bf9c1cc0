"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module draws random numbers and rounds them to the storage dtype; it holds
none of the attention arithmetic.  Recipe: a CPU ``torch.Generator`` seeded with
``seed`` draws fp32 N(0, 1) tensors of shape [B, H, N, d] in the order Q, K, V,
dO; Q and K are multiplied by ``qk_gain`` (4 for the long-context stress case);
every tensor is then rounded to ``dtype`` with round-to-nearest-even.  The
oracle receives the same rounded values upcast to float64, so input rounding is
not counted as kernel error.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, dtype, mask and input recipe."""

    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    dtype: torch.dtype = torch.bfloat16
    backward: bool = False
    qk_gain: float = 1.0
    sampled_rows: int = 0  # > 0: the oracle checks this many query rows per head

    @property
    def scale(self) -> float:
        return 1.0 / float(self.d) ** 0.5


# The five workloads of the method's task statement (shapes, dtypes, masks).
WORKLOADS = {
    "fwd_b1h1n256d64_fp32": Workload("fwd_b1h1n256d64_fp32", 1, 1, 256, 64, False, torch.float32),
    "fwd_b4h16n1024d64": Workload("fwd_b4h16n1024d64", 4, 16, 1024, 64, False),
    "fwd_b2h32n4096d128_causal": Workload("fwd_b2h32n4096d128_causal", 2, 32, 4096, 128, True),
    "fwdbwd_b2h16n2048d128_causal": Workload(
        "fwdbwd_b2h16n2048d128_causal", 2, 16, 2048, 128, True, backward=True
    ),
    "fwd_b1h8n32768d128_causal_x4": Workload(
        "fwd_b1h8n32768d128_causal_x4", 1, 8, 32768, 128, True, qk_gain=4.0, sampled_rows=512
    ),
}


def make_inputs(B, H, N, d, dtype=torch.bfloat16, seed=0, qk_gain=1.0, with_do=False):
    """Draw Q, K, V (and dO) as described in the module docstring (CPU tensors)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32) if with_do else None
    if qk_gain != 1.0:
        q.mul_(qk_gain)
        k.mul_(qk_gain)
    out = [q.to(dtype), k.to(dtype), v.to(dtype)]
    if with_do:
        out.append(do.to(dtype))
    return tuple(out)


E4M3_MAX = 448.0  # largest finite OCP FP8 E4M3 value


def make_fp8_inputs(B, H, N, d, seed=0, qk_gain=1.0, Hkv=None, Nk=None):
    """FP8 (e4m3) Q, K, V with one scale per tensor (CPU tensors).

    Q, K, V are drawn as in ``make_inputs`` (same seed, same order), then each
    tensor x is stored as e4m3(x / s) with s = amax(|x|) / 448, so its largest
    value lands on the top of the e4m3 range; s is returned as the tensor's
    descale (the stored values stand for s * stored).  With Hkv / Nk given, K and
    V are drawn with those head count and length from seed + 100.
    Returns (q8, k8, v8, q_descale, k_descale, v_descale)."""
    q = make_inputs(B, H, N, d, dtype=torch.float32, seed=seed, qk_gain=qk_gain)[0]
    if Hkv is None and Nk is None:
        k, v = make_inputs(B, H, N, d, dtype=torch.float32, seed=seed, qk_gain=qk_gain)[1:3]
    else:
        k, v = make_inputs(B, Hkv or H, Nk or N, d, dtype=torch.float32, seed=seed + 100,
                           qk_gain=qk_gain)[1:3]
    out, scales = [], []
    for x in (q, k, v):
        s = float(x.abs().max()) / E4M3_MAX
        s = s if s > 0 else 1.0
        out.append((x / s).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn))
        scales.append(s)
    return (*out, *scales)


def fp8_values(x8, descale):
    """The values an e4m3 tensor with a per-tensor descale stands for, float64 numpy."""
    return x8.to(torch.float64).numpy() * float(descale)


def sample_rows(N, count, seed, head):
    """Distinct query rows for one head: rows 0 and N-1 always, the rest uniform.

    ``numpy.random.default_rng(seed + head)`` draws ``count - 2`` distinct rows
    from 1..N-2; the result is sorted.  With count >= N every row is returned.
    """
    if count >= N:
        return np.arange(N, dtype=np.int64)
    rng = np.random.default_rng(int(seed) + int(head))
    mid = rng.choice(np.arange(1, N - 1), size=count - 2, replace=False)
    return np.sort(np.concatenate([[0, N - 1], mid]).astype(np.int64))


def to_f64(t):
    """A torch tensor (any dtype, any device) as a float64 numpy array."""
    return t.detach().to("cpu", torch.float64).numpy()
