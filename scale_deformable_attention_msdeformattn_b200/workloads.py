"""Seeded synthetic workloads for multi-scale deformable attention.

This module only *draws numbers*: it holds the five workload shapes and a
counter-based random generator, and none of the operator's arithmetic
(no bilinear sampling, no location mapping, no softmax).  Both the CUDA path's
tests and the fp64 oracle are fed from here, so neither side can bias the
inputs toward the other.

Generator (published methods, implemented here from their definitions):
  * SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014) used in counter form: draw i of stream s is
    mix64(s + (i + 1) * 0x9E3779B97F4A7C15).
  * uniform double in [0, 1) from the top 53 bits.
  * Box-Muller (1958) for normal deviates.

Each tensor has its own sub-stream; the stream seed is mix64(seed ^ tag).

Workload shapes follow the Deformable-DETR encoder / decoder settings the pages
describe (cf-1.com/news/4799680 §3.3: four flattened levels with strides
8/16/32/64, M=8 heads, K=4 points; discosf.com/news/5175395 §2.2: the
num_heads=8, num_levels=4, num_points=4 default).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# tags of the per-tensor sub-streams
TAG_VALUE = 1
TAG_REF = 2
TAG_OFFSETS = 3
TAG_LOGITS = 4
TAG_GRAD_OUT = 5
TAG_LOC_JITTER = 6
TAG_WEIGHTS = 7


def _mix64(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_seed(seed: int, tag: int) -> np.uint64:
    return _mix64(np.array([np.uint64(seed) ^ np.uint64(tag)], dtype=np.uint64))[0]


def splitmix64(seed: int, tag: int, n: int, offset: int = 0) -> np.ndarray:
    """Draws offset .. offset+n-1 of sub-stream (seed, tag) as uint64."""
    s = stream_seed(seed, tag)
    i = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = s + i * _GOLDEN
    return _mix64(z)


def uniform(seed: int, tag: int, n: int, offset: int = 0) -> np.ndarray:
    """Uniform doubles in [0, 1) (53-bit)."""
    u = splitmix64(seed, tag, n, offset) >> np.uint64(11)
    return u.astype(np.float64) * (1.0 / 9007199254740992.0)


def normal(seed: int, tag: int, n: int) -> np.ndarray:
    """n standard normal doubles by Box-Muller over pairs of uniforms."""
    npairs = (n + 1) // 2
    u = uniform(seed, tag, 2 * npairs)
    u1 = 1.0 - u[0::2]  # (0, 1]: log is finite
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * np.pi * u2
    out = np.empty(2 * npairs, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out[:n]


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Rounds to float32 (nearest-even), then to bfloat16 (nearest-even).

    Returns the raw uint16 bit patterns.  Finite inputs only."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = (b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns."""
    u = bits.astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int               # seed = 0x5EED0000 + index
    B: int
    levels: Tuple[Tuple[int, int], ...]   # (H, W) per level
    Q: Optional[int]         # None: encoder self-attention, Q = S
    M: int
    D: int
    K: int
    dtype: str               # value / output dtype: "f32", "bf16", "s8" or "e4m3" (one-byte value
                             # quantised from the bf16 draw; output, grad_output bf16)
    ref: str                 # "pixel_centre" | "uniform" | "uniform_inner"
    offset_sigma: float      # pixels of the sampled level
    logit_sigma: float

    @property
    def L(self) -> int:
        return len(self.levels)

    @property
    def S(self) -> int:
        return int(sum(h * w for h, w in self.levels))

    @property
    def num_queries(self) -> int:
        return self.S if self.Q is None else self.Q

    @property
    def seed(self) -> int:
        return 0x5EED0000 + self.index

    @property
    def samples(self) -> int:
        """Sampled points per pass: B * Q * M * L * K."""
        return self.B * self.num_queries * self.M * self.L * self.K

    def with_batch(self, B: int) -> "Workload":
        return dataclasses.replace(self, B=B)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_f32", 0, 1, ((8, 8), (4, 4)), 16, 2, 8, 2, "f32",
                 "uniform", 1.0, 1.0),
        Workload("detr_encoder_f32", 1, 1, ((100, 167), (50, 84), (25, 42), (13, 21)),
                 None, 8, 32, 4, "f32", "pixel_centre", 2.0, 1.0),
        Workload("detr_decoder_bf16", 2, 8, ((100, 167), (50, 84), (25, 42), (13, 21)),
                 300, 8, 32, 4, "bf16", "uniform_inner", 4.0, 1.0),
        Workload("encoder_1024_bf16", 3, 4, ((128, 128), (64, 64), (32, 32), (16, 16)),
                 None, 8, 32, 4, "bf16", "pixel_centre", 2.0, 1.0),
        Workload("stress_1080p_k8_bf16", 4, 2, ((135, 240), (68, 120), (34, 60), (17, 30)),
                 None, 8, 32, 8, "bf16", "pixel_centre", 8.0, 2.0),
        # INT8 value storage on the same draws as the two bf16 encoders above
        Workload("encoder_1024_s8", 3, 4, ((128, 128), (64, 64), (32, 32), (16, 16)),
                 None, 8, 32, 4, "s8", "pixel_centre", 2.0, 1.0),
        Workload("stress_1080p_k8_s8", 4, 2, ((135, 240), (68, 120), (34, 60), (17, 30)),
                 None, 8, 32, 8, "s8", "pixel_centre", 8.0, 2.0),
        # FP8 (E4M3) value storage on the same draws
        Workload("encoder_1024_e4m3", 3, 4, ((128, 128), (64, 64), (32, 32), (16, 16)),
                 None, 8, 32, 4, "e4m3", "pixel_centre", 2.0, 1.0),
        Workload("stress_1080p_k8_e4m3", 4, 2, ((135, 240), (68, 120), (34, 60), (17, 30)),
                 None, 8, 32, 8, "e4m3", "pixel_centre", 8.0, 2.0),
    ]
}


def custom(name: str, B: int, levels: List[Tuple[int, int]], Q: Optional[int], M: int,
           D: int, K: int, dtype: str = "f32", ref: str = "uniform",
           offset_sigma: float = 1.0, logit_sigma: float = 1.0, index: int = 100) -> Workload:
    """A small ad-hoc workload (tests use these for ragged and edge shapes)."""
    return Workload(name, index, B, tuple(tuple(x) for x in levels), Q, M, D, K, dtype, ref,
                    offset_sigma, logit_sigma)


def level_start_index(levels) -> np.ndarray:
    """Start of each level in the flattened key axis (input bookkeeping)."""
    sizes = [h * w for h, w in levels]
    return np.array([0] + list(np.cumsum(sizes)[:-1]), dtype=np.int64)


@dataclasses.dataclass
class Inputs:
    """All arrays are host numpy arrays in the operator's row-major layouts.

    value_bits is the stored value tensor: float32 array for "f32", uint16
    bfloat16 bit patterns for "bf16" and for "s8" / "e4m3" (the source that is
    then quantised to one byte).  Everything else is float32.
    """
    workload: Workload
    value: np.ndarray            # [B, S, M, D] float32 or uint16 (bf16 bits)
    spatial_shapes: np.ndarray   # [L, 2] int64 (H, W)
    level_start_index: np.ndarray  # [L] int64
    reference_points: np.ndarray   # [B, Q, 2] float32, normalized (x, y)
    sampling_offsets: np.ndarray   # [B, Q, M, L, K, 2] float32, level pixels
    attention_logits: np.ndarray   # [B, Q, M, L*K] float32
    grad_output: np.ndarray        # [B, Q, M, D] float32 or uint16 (bf16 bits)
    sampling_locations: np.ndarray  # [B, Q, M, L, K, 2] float32 (non-fused inputs)
    attention_weights: np.ndarray   # [B, Q, M, L, K] float32 (non-fused inputs)

    def value_f64(self) -> np.ndarray:
        return _widen(self.value)

    def grad_output_f64(self) -> np.ndarray:
        return _widen(self.grad_output)


def _widen(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return bf16_bits_to_f64(a)
    return a.astype(np.float64)


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype in ("bf16", "s8", "e4m3"):  # s8, e4m3: the bf16 source of the quantised value
        return to_bf16_bits(x)
    return x.astype(np.float32)


def reference_points(w: Workload) -> np.ndarray:
    """[B, Q, 2] normalized reference points following the workload's recipe."""
    B, Q = w.B, w.num_queries
    if w.ref == "pixel_centre":
        # encoder queries are the flattened tokens themselves; each sits at the
        # centre of its own pixel, in its own level's normalized frame
        pts = []
        for (h, wd) in w.levels:
            iy, ix = np.meshgrid(np.arange(h, dtype=np.float64), np.arange(wd, dtype=np.float64),
                                 indexing="ij")
            pts.append(np.stack([(ix.ravel() + 0.5) / wd, (iy.ravel() + 0.5) / h], -1))
        one = np.concatenate(pts, 0)
        assert one.shape[0] == Q
        return np.broadcast_to(one, (B, Q, 2)).astype(np.float64)
    u = uniform(w.seed, TAG_REF, B * Q * 2).reshape(B, Q, 2)
    if w.ref == "uniform_inner":
        return 0.05 + 0.9 * u
    return u


def generate(w: Workload, with_nonfused: bool = True) -> Inputs:
    """Draws every input of one pass of the workload (deterministic in w.seed)."""
    B, S, Q, M, D, L, K = w.B, w.S, w.num_queries, w.M, w.D, w.L, w.K
    value = normal(w.seed, TAG_VALUE, B * S * M * D).reshape(B, S, M, D)
    ref = reference_points(w)
    off = (w.offset_sigma * normal(w.seed, TAG_OFFSETS, B * Q * M * L * K * 2)
           ).reshape(B, Q, M, L, K, 2)
    logits = (w.logit_sigma * normal(w.seed, TAG_LOGITS, B * Q * M * L * K)
              ).reshape(B, Q, M, L * K)
    gout = normal(w.seed, TAG_GRAD_OUT, B * Q * M * D).reshape(B, Q, M, D)
    shapes = np.array(w.levels, dtype=np.int64).reshape(L, 2)
    if with_nonfused:
        # inputs of the non-fused operator, drawn directly: a location is the
        # reference point plus Gaussian jitter of offset_sigma level-pixels
        # (expressed in that level's normalized units); weights are a flat
        # Dirichlet draw (normalized unit exponentials) over the L*K points
        jit = normal(w.seed, TAG_LOC_JITTER, B * Q * M * L * K * 2).reshape(B, Q, M, L, K, 2)
        scale = np.stack([1.0 / shapes[:, 1], 1.0 / shapes[:, 0]], -1).astype(np.float64)
        loc = ref[:, :, None, None, None, :] + w.offset_sigma * jit * scale[None, None, None, :, None, :]
        e = -np.log(1.0 - uniform(w.seed, TAG_WEIGHTS, B * Q * M * L * K)).reshape(B, Q, M, L * K)
        e = np.maximum(e, 1e-30)
        wts = (e / e.sum(-1, keepdims=True)).reshape(B, Q, M, L, K)
    else:
        loc = np.zeros((0,), np.float64)
        wts = np.zeros((0,), np.float64)
    return Inputs(
        workload=w,
        value=_store(value, w.dtype),
        spatial_shapes=shapes,
        level_start_index=level_start_index(w.levels),
        reference_points=np.ascontiguousarray(ref, dtype=np.float32),
        sampling_offsets=off.astype(np.float32),
        attention_logits=logits.astype(np.float32),
        grad_output=_store(gout, w.dtype),
        sampling_locations=np.ascontiguousarray(loc, dtype=np.float32),
        attention_weights=np.ascontiguousarray(wts, dtype=np.float32),
    )


# ----------------------------------------------------------- DCNv3 core ----
#
# Stand-ins for InternImage's DCNv3 layers (discosf.com/news/5175395 §4.2 gives
# the operator and mentions 7x7 and larger kernels, but no layer sizes): a
# classification stage-1 layer at 224^2 input (56 x 56, 64 channels in 4
# groups), a detection stage-2 layer at 800 x 1333 (100 x 167, 128 channels in
# 8 groups) and a 7 x 7 large-kernel layer.  Offsets are N(0, sigma) pixels,
# masks a flat Dirichlet draw over the K points of each (n, i, j, g).

@dataclasses.dataclass(frozen=True)
class DcnWorkload:
    name: str
    index: int               # seed = 0x5EED0000 + index
    N: int
    H: int
    W: int
    G: int
    C: int
    kernel: Tuple[int, int]
    stride: Tuple[int, int]
    pad: Tuple[int, int]
    dil: Tuple[int, int]
    dtype: str               # "f32", "bf16" or "s8" (as Workload.dtype)
    offset_sigma: float

    @property
    def seed(self) -> int:
        return 0x5EED0000 + self.index

    @property
    def K(self) -> int:
        return self.kernel[0] * self.kernel[1]

    @property
    def out_hw(self) -> Tuple[int, int]:
        kh, kw = self.kernel
        return ((self.H + 2 * self.pad[0] - self.dil[0] * (kh - 1) - 1) // self.stride[0] + 1,
                (self.W + 2 * self.pad[1] - self.dil[1] * (kw - 1) - 1) // self.stride[1] + 1)

    @property
    def samples(self) -> int:
        Ho, Wo = self.out_hw
        return self.N * Ho * Wo * self.G * self.K


DCN_WORKLOADS: Dict[str, DcnWorkload] = {
    w.name: w
    for w in [
        DcnWorkload("dcnv3_stage1_f32", 10, 32, 56, 56, 4, 16, (3, 3), (1, 1), (1, 1), (1, 1),
                    "f32", 1.0),
        DcnWorkload("dcnv3_det_stage2_bf16", 11, 2, 100, 167, 8, 16, (3, 3), (1, 1), (1, 1), (1, 1),
                    "bf16", 1.0),
        DcnWorkload("dcnv3_k7_bf16", 12, 2, 50, 84, 16, 16, (7, 7), (1, 1), (3, 3), (1, 1),
                    "bf16", 2.0),
    ]
}

TAG_DCN_MASK = 8


@dataclasses.dataclass
class DcnInputs:
    workload: DcnWorkload
    input: np.ndarray        # [N, H, W, G, C] float32, or bf16 bits (uint16) for bf16 / s8
    offset: np.ndarray       # [N, Ho, Wo, G, K, 2] float32 (dx, dy) pixels
    mask: np.ndarray         # [N, Ho, Wo, G, K] float32
    grad_output: np.ndarray  # [N, Ho, Wo, G, C] float32 or bf16 bits

    def input_f64(self) -> np.ndarray:
        return _widen(self.input)

    def grad_output_f64(self) -> np.ndarray:
        return _widen(self.grad_output)


def generate_dcn(w: DcnWorkload) -> DcnInputs:
    N, H, W, G, C, K = w.N, w.H, w.W, w.G, w.C, w.K
    Ho, Wo = w.out_hw
    x = normal(w.seed, TAG_VALUE, N * H * W * G * C).reshape(N, H, W, G, C)
    off = (w.offset_sigma * normal(w.seed, TAG_OFFSETS, N * Ho * Wo * G * K * 2)
           ).reshape(N, Ho, Wo, G, K, 2)
    e = -np.log(1.0 - uniform(w.seed, TAG_DCN_MASK, N * Ho * Wo * G * K)).reshape(N, Ho, Wo, G, K)
    e = np.maximum(e, 1e-30)
    mask = e / e.sum(-1, keepdims=True)
    gy = normal(w.seed, TAG_GRAD_OUT, N * Ho * Wo * G * C).reshape(N, Ho, Wo, G, C)
    return DcnInputs(w, _store(x, w.dtype), off.astype(np.float32), mask.astype(np.float32),
                     _store(gy, w.dtype))


def custom_dcn(name: str, N: int, H: int, W: int, G: int, C: int, kernel, stride=(1, 1),
               pad=(1, 1), dil=(1, 1), dtype: str = "f32", offset_sigma: float = 1.0,
               index: int = 700) -> DcnWorkload:
    """A small ad-hoc DCNv3 workload (tests)."""
    return DcnWorkload(name, index, N, H, W, G, C, tuple(kernel), tuple(stride), tuple(pad),
                       tuple(dil), dtype, offset_sigma)
