"""The five synthetic MoE-layer workloads, as plain data.

Each workload names the layer shape (H hidden, I expert intermediate, E experts,
k chosen per token, L layers), the FP4 weight format, how the weights and the
routing skew are drawn, the batch sizes, the number of decode steps and the size
of the HBM expert-slot pool.  Nothing here computes any part of the MoE layer.

Shapes follow the models the FreeToken write-ups name: a 35B-A3B MoE with NVFP4
experts and a 284B MoE (256 experts, 6 active) with MXFP4 experts
(post.smzdm.com/p/a825qpgl, sections 一 and 二).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

MXFP4 = "mxfp4"
NVFP4 = "nvfp4"

GIB = 1 << 30


@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    I: int
    E: int
    k: int
    L: int
    fmt: str
    seed: int
    batches: tuple
    steps: int
    zipf_s: float
    # weights: "uniform" = uniform E2M1 nibbles + E8M0 exponents in exp_range;
    # "normal" = N(0, sigma) floats quantised to NVFP4
    weight_recipe: str
    exp_range: tuple = (0, 0)
    sigma: float = 0.02
    # single layer repeated: every layer position reuses layer 0's parameters
    shared_layer: bool = False
    # slot pool size: a fraction of L*E experts, or a byte cap, or None = all resident
    slot_frac: float | None = None
    slot_bytes_cap: int | None = None
    renormalize: int = 1
    notes: str = field(default="", compare=False)


TINY = Workload(
    name="tiny_h256_e16_k2", H=256, I=256, E=16, k=2, L=1, fmt=MXFP4, seed=0,
    batches=(4,), steps=1, zipf_s=0.0, weight_recipe="uniform", exp_range=(-4, 0),
    notes="single tiny layer, all experts resident")

DECODE_35B = Workload(
    name="decode_35b_a3b_h2048_e128_k8", H=2048, I=768, E=128, k=8, L=48, fmt=NVFP4,
    seed=2, batches=(1, 4, 8), steps=256, zipf_s=1.1, weight_recipe="normal",
    sigma=0.02, shared_layer=True, slot_frac=0.25,
    notes="one layer's parameters repeated at 48 layer positions; 25% of L*E experts fit in HBM")

DECODE_284B = Workload(
    name="decode_284b_h4096_e256_k6", H=4096, I=2048, E=256, k=6, L=40, fmt=MXFP4,
    seed=3, batches=(1,), steps=128, zipf_s=1.0, weight_recipe="uniform",
    exp_range=(-10, -6), slot_bytes_cap=32 * GIB,
    notes="Zipf permutation re-drawn per layer; slot pool capped at 32 GiB")

PREFILL_35B = Workload(
    name="prefill_35b_a3b_t2048", H=2048, I=768, E=128, k=8, L=1, fmt=NVFP4, seed=2,
    batches=(2048,), steps=1, zipf_s=0.0, weight_recipe="normal", sigma=0.02,
    notes="2048-token prompt on the decode_35b layer (same weights), no routing bias, "
          "all experts resident")

STRESS_284B = Workload(
    name="stress_284b", H=4096, I=2048, E=256, k=6, L=40, fmt=MXFP4, seed=5,
    batches=(1,), steps=64, zipf_s=1.0, weight_recipe="uniform", exp_range=(-10, -6),
    slot_frac=0.25, notes="swept over zipf_s and slot_frac")

STRESS_ZIPF = (0.0, 0.6, 1.0, 1.4)
STRESS_POOL = (0.10, 0.25, 0.50)

# (B_pcie, B_host) GB/s pairs of the four machines in the bandwidth table of
# post.smzdm.com/p/a825qpgl section 二
QSTAR_MACHINES = ((49.0, 53.8), (52.7, 77.3), (25.1, 63.2), (11.8, 47.5))

ALL = {w.name: w for w in (TINY, DECODE_35B, DECODE_284B, PREFILL_35B, STRESS_284B)}


def stress_variant(zipf_s: float, pool_frac: float) -> Workload:
    return replace(STRESS_284B, name=f"stress_284b_s{zipf_s:g}_p{int(pool_frac * 100)}",
                   zipf_s=zipf_s, slot_frac=pool_frac)


def block_elems(fmt: str) -> int:
    """Elements sharing one block scale: 32 for MXFP4, 16 for NVFP4."""
    return 32 if fmt == MXFP4 else 16


def align4k(n: int) -> int:
    return (n + 4095) & ~4095


def expert_block_bytes(w: Workload) -> int:
    """Bytes of one expert in the 4096-aligned host/slot layout (6 tensors)."""
    bs = block_elems(w.fmt)
    gu = align4k(w.I * w.H // 2) + align4k(w.I * w.H // bs)
    dn = align4k(w.H * w.I // 2) + align4k(w.H * w.I // bs)
    return 2 * gu + dn


def n_slots(w: Workload) -> int:
    total = w.L * w.E
    if w.slot_frac is not None:
        return max(1, int(round(w.slot_frac * total)))
    if w.slot_bytes_cap is not None:
        return min(total, w.slot_bytes_cap // expert_block_bytes(w))
    return total
