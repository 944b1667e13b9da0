"""Seeded synthetic inputs for the dequant GEMV: weight bytes and fp16 activations.

This module holds none of the GEMV's arithmetic: it only draws random numbers and places bytes.
Both the CUDA path and the CPU oracle consume what it produces.

Q4_K superblock bytes (144 per 256 weights): bytes 0-1 = fp16 d ~ U(1e-4, 2e-3), bytes 2-3 =
fp16 dmin ~ U(0, 1e-3) (each drawn in fp64 and rounded once to fp16), bytes 4-143 uniform random.
Uniform bytes 4-15 are exactly uniform 6-bit (sc_j, m_j) for all eight sub-blocks, because the GGML
scale table packs the 96 bits of eight (sc, m) pairs into the 12 bytes one-to-one; uniform bytes
16-143 are exactly uniform 4-bit q for all 256 weights.  (The one-to-one packing is checked by the
oracle tests.)

Q8_0 block bytes (34 per 32 weights): bytes 0-1 = fp16 d ~ U(1e-3, 1e-2), bytes 2-33 = int8 q
uniform on -127..127 (-128 is never drawn).

Q5_K superblock bytes (176 per 256 weights): d and dmin as for Q4_K (bytes 0-3), bytes 4-175
uniform random: uniform (sc, m) as for Q4_K, and uniform 5-bit q (qh and qs together hold each
weight's five bits once).

Q6_K superblock bytes (210 per 256 weights): bytes 0-207 uniform random (uniform 6-bit q, stored
q - 32 in -32..31, and uniform int8 scales per 16 weights), bytes 208-209 = fp16 d ~ U(1e-5, 2e-4).

IQ4_XS superblock bytes (136 per 256 weights): bytes 0-1 = fp16 d ~ U(2e-5, 2e-4), bytes 2-135
uniform random: uniform 6-bit sub-block scales (scales_h and scales_l hold each scale's six bits
once) and uniform 4-bit codebook indices.

Activations: x fp16 [K, B] with entries N(0, 1) drawn in fp64 and rounded once to fp16; for the
"massive activation" FFN inputs each entry is independently, with probability 1e-3, multiplied by
100 before that rounding.

Streams: every tensor gets its own PCG64 stream keyed by (seed, tensor id, purpose), purpose 0 for
weights and 1 for activations.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

Q8_0 = 8
Q4_K = 12
Q5_K = 13
Q6_K = 14
IQ4_XS = 23

BLOCK_WEIGHTS = {Q4_K: 256, Q8_0: 32, Q5_K: 256, Q6_K: 256, IQ4_XS: 256}
BLOCK_BYTES = {Q4_K: 144, Q8_0: 34, Q5_K: 176, Q6_K: 210, IQ4_XS: 136}


def _rng(seed: int, tensor_id: int, purpose: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id, purpose])))


def weight_bytes(fmt: int, N: int, K: int) -> int:
    return N * (K // BLOCK_WEIGHTS[fmt]) * BLOCK_BYTES[fmt]


def q4k_weights(N: int, K: int, seed: int, tensor_id: int = 0,
                d_range=(1e-4, 2e-3), dmin_range=(0.0, 1e-3)) -> np.ndarray:
    """Random Q4_K tensor [N, K] as raw bytes (uint8, N*K/256*144)."""
    assert K % 256 == 0
    g = _rng(seed, tensor_id, 0)
    nsb = N * (K // 256)
    blk = g.integers(0, 256, size=(nsb, 144), dtype=np.uint8)
    d = g.uniform(d_range[0], d_range[1], size=nsb).astype(np.float16)
    dmin = g.uniform(dmin_range[0], dmin_range[1], size=nsb).astype(np.float16)
    blk[:, 0:2] = d.view(np.uint8).reshape(nsb, 2)
    blk[:, 2:4] = dmin.view(np.uint8).reshape(nsb, 2)
    return blk.reshape(-1)


def q8_0_weights(N: int, K: int, seed: int, tensor_id: int = 0,
                 d_range=(1e-3, 1e-2)) -> np.ndarray:
    """Random Q8_0 tensor [N, K] as raw bytes (uint8, N*K/32*34)."""
    assert K % 32 == 0
    g = _rng(seed, tensor_id, 0)
    nblk = N * (K // 32)
    blk = np.empty((nblk, 34), dtype=np.uint8)
    d = g.uniform(d_range[0], d_range[1], size=nblk).astype(np.float16)
    q = g.integers(-127, 128, size=(nblk, 32), dtype=np.int8)
    blk[:, 0:2] = d.view(np.uint8).reshape(nblk, 2)
    blk[:, 2:34] = q.view(np.uint8)
    return blk.reshape(-1)


def q5k_weights(N: int, K: int, seed: int, tensor_id: int = 0,
                d_range=(1e-4, 2e-3), dmin_range=(0.0, 1e-3)) -> np.ndarray:
    """Random Q5_K tensor [N, K] as raw bytes (uint8, N*K/256*176)."""
    assert K % 256 == 0
    g = _rng(seed, tensor_id, 0)
    nsb = N * (K // 256)
    blk = g.integers(0, 256, size=(nsb, 176), dtype=np.uint8)
    d = g.uniform(d_range[0], d_range[1], size=nsb).astype(np.float16)
    dmin = g.uniform(dmin_range[0], dmin_range[1], size=nsb).astype(np.float16)
    blk[:, 0:2] = d.view(np.uint8).reshape(nsb, 2)
    blk[:, 2:4] = dmin.view(np.uint8).reshape(nsb, 2)
    return blk.reshape(-1)


def q6k_weights(N: int, K: int, seed: int, tensor_id: int = 0, d_range=(1e-5, 2e-4)) -> np.ndarray:
    """Random Q6_K tensor [N, K] as raw bytes (uint8, N*K/256*210)."""
    assert K % 256 == 0
    g = _rng(seed, tensor_id, 0)
    nsb = N * (K // 256)
    blk = g.integers(0, 256, size=(nsb, 210), dtype=np.uint8)
    d = g.uniform(d_range[0], d_range[1], size=nsb).astype(np.float16)
    blk[:, 208:210] = d.view(np.uint8).reshape(nsb, 2)
    return blk.reshape(-1)


def iq4xs_weights(N: int, K: int, seed: int, tensor_id: int = 0, d_range=(2e-5, 2e-4)) -> np.ndarray:
    """Random IQ4_XS tensor [N, K] as raw bytes (uint8, N*K/256*136)."""
    assert K % 256 == 0
    g = _rng(seed, tensor_id, 0)
    nsb = N * (K // 256)
    blk = g.integers(0, 256, size=(nsb, 136), dtype=np.uint8)
    d = g.uniform(d_range[0], d_range[1], size=nsb).astype(np.float16)
    blk[:, 0:2] = d.view(np.uint8).reshape(nsb, 2)
    return blk.reshape(-1)


def weights(fmt: int, N: int, K: int, seed: int, tensor_id: int = 0) -> np.ndarray:
    if fmt == Q4_K:
        return q4k_weights(N, K, seed, tensor_id)
    if fmt == Q8_0:
        return q8_0_weights(N, K, seed, tensor_id)
    if fmt == Q5_K:
        return q5k_weights(N, K, seed, tensor_id)
    if fmt == Q6_K:
        return q6k_weights(N, K, seed, tensor_id)
    if fmt == IQ4_XS:
        return iq4xs_weights(N, K, seed, tensor_id)
    raise ValueError(f"unknown format {fmt}")


def activations(K: int, B: int, seed: int, tensor_id: int = 0,
                massive_frac: float = 0.0, massive_scale: float = 100.0) -> np.ndarray:
    """fp16 x [K, B] ~ N(0, 1); with massive_frac > 0 that fraction of entries is scaled first."""
    g = _rng(seed, tensor_id, 1)
    v = g.standard_normal(size=(K, B))
    if massive_frac > 0.0:
        hit = g.random(size=(K, B)) < massive_frac
        v = np.where(hit, v * massive_scale, v)
    return v.astype(np.float16)


@dataclass(frozen=True)
class Gemv:
    """One GEMV call of a workload: format, shape, columns and the tensor id of its inputs."""
    name: str
    fmt: int
    N: int
    K: int
    B: int = 1
    tensor_id: int = 0
    massive_frac: float = 0.0

    @property
    def weight_bytes(self) -> int:
        return weight_bytes(self.fmt, self.N, self.K)

    @property
    def algorithmic_bytes(self) -> int:
        """Weight bytes + fp16 x bytes + fp32 y bytes: what one call must move at least once."""
        return self.weight_bytes + 2 * self.K * self.B + 4 * self.N * self.B


@dataclass(frozen=True)
class Workload:
    """A named list of GEMV calls that share a seed (issued in order on one stream)."""
    name: str
    seed: int
    calls: tuple = field(default_factory=tuple)

    def inputs(self, call: Gemv):
        W = weights(call.fmt, call.N, call.K, self.seed, call.tensor_id)
        x = activations(call.K, call.B, self.seed, call.tensor_id, call.massive_frac)
        return W, x


# The decode-time weight shapes of a 27B-class hybrid (Gated DeltaNet + GQA) model, hidden size
# 5120, FFN size 17408, as listed in the T4 hardware/model dossier (tensor shapes, quant mix).
WORKLOADS = {
    # attn_k / attn_v projection (4 KV heads x 256), seed 0
    "q4k_attn_kv_1024x5120": Workload("q4k_attn_kv_1024x5120", 0, (
        Gemv("attn_kv", Q4_K, 1024, 5120, 1, 0),)),
    # DeltaNet fused QKV projection
    "q4k_ssm_qkv_10240x5120": Workload("q4k_ssm_qkv_10240x5120", 1, (
        Gemv("attn_qkv", Q4_K, 10240, 5120, 1, 0),)),
    # FFN gate/up and down at B=1, activations with 0.1% entries scaled x100
    "q4k_ffn_pair_b1": Workload("q4k_ffn_pair_b1", 2, (
        Gemv("ffn_gate", Q4_K, 17408, 5120, 1, 0, 1e-3),
        Gemv("ffn_down", Q4_K, 5120, 17408, 1, 1, 1e-3))),
    # mixed-format call list: attention Q in Q8_0, then the SSM out-projection in Q4_K
    "mixed_q8_0_q4k_b1": Workload("mixed_q8_0_q4k_b1", 3, (
        Gemv("attn_q", Q8_0, 12288, 5120, 1, 0),
        Gemv("ssm_out", Q4_K, 5120, 6144, 1, 1))),
    # batched verify of up to 8 draft tokens on the FFN gate
    "q4k_ffn_gate_verify": Workload("q4k_ffn_gate_verify", 4, tuple(
        Gemv(f"ffn_gate_b{b}", Q4_K, 17408, 5120, b, 0) for b in (1, 2, 4, 8))),
    # the other K-quants of the dossier's quant mix on the same FFN tensors
    "q5k_ffn_pair_b1": Workload("q5k_ffn_pair_b1", 5, (
        Gemv("ffn_gate", Q5_K, 17408, 5120, 1, 0, 1e-3),
        Gemv("ffn_down", Q5_K, 5120, 17408, 1, 1, 1e-3))),
    "q6k_ffn_pair_b1": Workload("q6k_ffn_pair_b1", 6, (
        Gemv("ffn_gate", Q6_K, 17408, 5120, 1, 0, 1e-3),
        Gemv("ffn_down", Q6_K, 5120, 17408, 1, 1, 1e-3))),
    "kquant_ffn_gate_b8": Workload("kquant_ffn_gate_b8", 7, (
        Gemv("q5k_ffn_gate_b8", Q5_K, 17408, 5120, 8, 0),
        Gemv("q6k_ffn_gate_b8", Q6_K, 17408, 5120, 8, 1))),
    # the IQ4_XS row of the same FFN tensors (the T4 dossier's GEMV prompt names it next to Q4_K)
    "iq4xs_ffn_pair_b1": Workload("iq4xs_ffn_pair_b1", 8, (
        Gemv("ffn_gate", IQ4_XS, 17408, 5120, 1, 0, 1e-3),
        Gemv("ffn_down", IQ4_XS, 5120, 17408, 1, 1, 1e-3))),
    # verify widths beyond 8 (up to 16 draft tokens) on the FFN gate in every K-quant
    "kquant_ffn_gate_b16": Workload("kquant_ffn_gate_b16", 9, (
        Gemv("q4k_ffn_gate_b16", Q4_K, 17408, 5120, 16, 0),
        Gemv("q5k_ffn_gate_b16", Q5_K, 17408, 5120, 16, 1),
        Gemv("q6k_ffn_gate_b16", Q6_K, 17408, 5120, 16, 2))),
    # IQ4_XS on the batched-verify widths (the tensor-core kernel at B >= 2)
    "iq4xs_ffn_gate_verify": Workload("iq4xs_ffn_gate_verify", 10, (
        Gemv("ffn_gate_b2", IQ4_XS, 17408, 5120, 2, 0, 1e-3),
        Gemv("ffn_gate_b8", IQ4_XS, 17408, 5120, 8, 1, 1e-3),
        Gemv("ffn_gate_b16", IQ4_XS, 17408, 5120, 16, 2, 1e-3))),
    # the Q8_0 attention projection on the batched-verify widths (tensor cores at B >= 2)
    "q8_0_attn_q_verify": Workload("q8_0_attn_q_verify", 11, (
        Gemv("attn_q_b2", Q8_0, 12288, 5120, 2, 0),
        Gemv("attn_q_b8", Q8_0, 12288, 5120, 8, 1),
        Gemv("attn_q_b16", Q8_0, 12288, 5120, 16, 2))),
}
FMT_NAMES = {Q4_K: "Q4_K", Q5_K: "Q5_K", Q6_K: "Q6_K", Q8_0: "Q8_0", IQ4_XS: "IQ4_XS"}
