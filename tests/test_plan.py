"""Host-side tests of the launch planner through qg_plan (no GPU: the device limits are passed in).

The pinned choices are the slice counts that sweeps of forced slice counts measured fastest (or
within 0.2 us of the fastest) on a B200 (148 SMs, 232,448 bytes of opt-in shared memory per block)
for the decoder's GEMV shapes; the invariants hold for any shape and device size."""
import pytest

import quant_dequant_gemv_q4_b200 as qg
from quant_dequant_gemv_q4_b200 import synth

Q4_K, Q5_K, Q6_K, Q8_0 = synth.Q4_K, synth.Q5_K, synth.Q6_K, synth.Q8_0
IQ4_XS = synth.IQ4_XS
B200 = dict(sms=148, smem_optin=232448)
FACTORED, GENERIC, TENSOR, DIRECT = (qg.QG_VARIANT_FACTORED, qg.QG_VARIANT_GENERIC,
                                     qg.QG_VARIANT_TENSOR, qg.QG_VARIANT_DIRECT)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from quant_dequant_gemv_q4_b200 import build
    build.build()
    qg.lib()


@pytest.mark.parametrize("fmt,N,K,B,mats,variant,splits,warps", [
    (Q4_K, 17408, 5120, 1, 1, FACTORED, 1, 16),   # ffn_gate (the headline call)
    (Q4_K, 5120, 17408, 1, 1, FACTORED, 7, 16),   # ffn_down: 7 slices (12.7 us; 4 slices: 14.4)
    (Q4_K, 10240, 5120, 1, 1, FACTORED, 1, 16),   # attn_qkv: one slice (9.9 us; 2 slices: 10.5)
    (Q4_K, 5120, 6144, 1, 1, FACTORED, 4, 16),    # ssm_out
    (Q4_K, 1024, 5120, 1, 1, FACTORED, 4, 16),    # attn_k / attn_v
    (Q5_K, 5120, 17408, 1, 1, FACTORED, 7, 16),
    (Q6_K, 17408, 5120, 1, 1, FACTORED, 1, 12),
    (Q6_K, 5120, 17408, 1, 1, FACTORED, 5, 12),   # 29.6 us; 4 slices: 35.4
    (Q8_0, 12288, 5120, 1, 1, FACTORED, 3, 8),    # attn_q: 3 slices (13.8 us; one slice: 14.4)
    (Q8_0, 17408, 5120, 1, 1, FACTORED, 1, 8),
    (Q4_K, 17408, 5120, 2, 1, TENSOR, 1, 16),
    (Q4_K, 17408, 5120, 8, 1, TENSOR, 1, 12),
    (Q4_K, 5120, 17408, 8, 1, TENSOR, 5, 12),     # 20.1 us; 4 slices: 22.1
    (Q4_K, 10240, 5120, 8, 1, TENSOR, 1, 12),     # 14.1 us; 2 slices: 15.1
    (Q4_K, 17408, 5120, 16, 1, TENSOR, 2, 8),
    (Q6_K, 17408, 5120, 8, 1, TENSOR, 2, 8),
    (Q4_K, 17408, 5120, 1, 2, FACTORED, 1, 16),   # gate/up pair
    (Q4_K, 17408, 5120, 8, 2, TENSOR, 1, 12),
])
def test_measured_choices(fmt, N, K, B, mats, variant, splits, warps):
    p = qg.qg_plan(fmt, N, K, B, 0, mats, **B200)
    assert p["variant"] == variant
    assert p["splits"] == splits
    assert p["warps"] == warps
    assert p["ctas"] <= B200["sms"]
    assert p["smem"] <= B200["smem_optin"]


def test_headline_plan_in_full():
    assert qg.qg_plan(Q4_K, 17408, 5120, 1, **B200) == dict(
        variant=FACTORED, splits=1, units_per_slice=20, ctas=148, warps=16,
        smem=16 * 2 * 32 * 144 + 20 * (512 + 32) + 16 * 32 * 4 + 16 * 2 * 8)


SHAPES = [(1, 256), (17, 256), (33, 512), (100, 768), (1000, 2560), (4096, 4096), (1024, 5120),
          (5120, 6144), (10240, 5120), (17408, 5120), (5120, 17408), (40, 65536), (3, 131072)]


@pytest.mark.parametrize("sms,smem", [(148, 232448), (132, 232448), (8, 232448), (148, 180000)])
@pytest.mark.parametrize("fmt", [Q4_K, Q5_K, Q6_K, Q8_0, IQ4_XS])
def test_plan_invariants(sms, smem, fmt):
    """Every plan fits the device, covers K exactly once with its slices, launches at most one CTA
    per SM, and takes the variant qg_gemv's default rule names."""
    n = 0
    for N, K in SHAPES:
        UPR = K // 256
        for B in (1, 2, 3, 8, 16):
            for mats in (1, 2):
                try:
                    p = qg.qg_plan(fmt, N, K, B, 0, mats, sms, smem)
                except qg.QgError as e:
                    # B > 8 is the tensor-core kernels' only (not the Q6_K pair's, and IQ4_XS's
                    # with an even K / 256); a small device may fit no plan
                    wide_ok = fmt in (Q4_K, Q5_K, Q8_0) or (fmt == Q6_K and mats == 1) or \
                        (fmt == IQ4_XS and UPR % 2 == 0)
                    assert (B > 8 and not wide_ok and e.status == qg.QG_ERR_BATCH) or \
                        e.status == qg.QG_ERR_SHAPE, (N, K, B, mats, e)
                    continue
                n += 1
                S, US = p["splits"], p["units_per_slice"]
                assert p["smem"] <= smem
                assert S * US >= UPR > (S - 1) * US
                assert 1 <= p["ctas"] <= sms
                assert p["warps"] in (6, 8, 12, 16)
                has_tc = fmt in (Q4_K, Q5_K, Q6_K, Q8_0) or (fmt == IQ4_XS and UPR % 2 == 0)
                tc_min = 3 if fmt == Q6_K else 2  # Q6_K's CUDA-core kernel still wins at B = 2
                assert p["variant"] == (TENSOR if has_tc and B >= tc_min else FACTORED)
    assert n > 0


def test_less_shared_memory_means_more_slices():
    big = qg.qg_plan(Q4_K, 40, 65536, 1, **B200)
    assert big["splits"] > 1  # x of a 65536-long row does not fit next to the ring
    assert qg.qg_plan(Q4_K, 5120, 17408, 1, 0, 1, 148, 180000)["splits"] >= \
        qg.qg_plan(Q4_K, 5120, 17408, 1, **B200)["splits"]


def test_generic_and_direct_plans():
    p = qg.qg_plan(Q8_0, 300, 5152, 1, **B200)  # K not a multiple of 256: the per-row kernel
    assert p["variant"] == GENERIC and p["splits"] == 1 and p["units_per_slice"] == 5152 // 32
    d = qg.qg_plan(Q4_K, 17408, 5120, 1, DIRECT, **B200)
    assert d["variant"] == DIRECT and d["smem"] <= B200["smem_optin"]


@pytest.mark.parametrize("args,status", [
    ((7, 100, 5120, 1, 0, 1), qg.QG_ERR_FMT),
    ((Q4_K, 100, 5000, 1, 0, 1), qg.QG_ERR_SHAPE),
    ((Q4_K, 0, 5120, 1, 0, 1), qg.QG_ERR_SHAPE),
    ((Q4_K, 100, 5120, 0, 0, 1), qg.QG_ERR_BATCH),
    ((Q4_K, 100, 5120, 17, 0, 1), qg.QG_ERR_BATCH),
    ((Q8_0, 100, 5152, 9, 0, 1), qg.QG_ERR_BATCH),   # K % 256 != 0: no tensor-core kernel
    ((Q4_K, 100, 5120, 9, FACTORED, 1), qg.QG_ERR_BATCH),
    ((Q4_K, 100, 5120, 1, 9, 1), qg.QG_ERR_VARIANT),
    ((Q8_0, 100, 5152, 2, TENSOR, 1), qg.QG_ERR_VARIANT),
    ((Q8_0, 100, 5152, 1, FACTORED, 1), qg.QG_ERR_VARIANT),
    ((Q5_K, 100, 5120, 1, DIRECT, 1), qg.QG_ERR_VARIANT),
    ((Q4_K, 100, 5120, 1, FACTORED, 2), qg.QG_ERR_VARIANT),
    ((Q4_K, 100, 5120, 1, 0, 3), qg.QG_ERR_SHAPE),
    ((Q8_0, 100, 5152, 1, 0, 2), qg.QG_ERR_SHAPE),
])
def test_argument_errors(args, status):
    with pytest.raises(qg.QgError) as e:
        qg.qg_plan(*args, **B200)
    assert e.value.status == status


def test_null_out():
    assert qg.lib().qg_plan(Q4_K, 100, 5120, 1, 0, 1, 148, 232448, None) == qg.QG_ERR_NULL


@pytest.mark.parametrize("wl", sorted(synth.WORKLOADS))
def test_every_workload_call_has_a_plan(wl):
    """Every call of the synthetic workloads (the parity configurations and the bench table) plans
    on a B200 with the default variant, and the variant is the one the default rule names."""
    for c in synth.WORKLOADS[wl].calls:
        p = qg.qg_plan(c.fmt, c.N, c.K, c.B, **B200)
        assert p["smem"] <= B200["smem_optin"] and 1 <= p["ctas"] <= B200["sms"]
        UPR = c.K // 256
        has_tc = c.fmt in (Q4_K, Q5_K, Q6_K, Q8_0) or (c.fmt == IQ4_XS and UPR % 2 == 0)
        tc_min = 3 if c.fmt == Q6_K else 2
        assert p["variant"] == (TENSOR if has_tc and c.B >= tc_min else FACTORED), (wl, c.name)
