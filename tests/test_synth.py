"""The seeded input generator: published splitmix64 vectors, one correct BF16
rounding, the workload recipes' shapes and value distributions."""

import numpy as np
import pytest
import torch

import fqa_synth as s


def test_splitmix64_published_vectors():
    # splitmix64 from state 0: the reference outputs published with the
    # generator (Steele, Lea, Flood 2014; also Vigna's splitmix64.c).
    u = s.mix64(np.arange(1, 4, dtype=np.uint64) * s.GAMMA)
    assert [int(x) for x in u] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_uniform_and_normal_moments():
    key = s.stream_key(7, 0, 0, 0)
    u = s.uniforms(key, 0, 1 << 20)
    assert 0.0 <= u.min() and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 2e-3
    z = s.normals(key, 1 << 20)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1.0) < 5e-3
    # distinct streams differ
    assert not np.array_equal(s.normals(s.stream_key(7, 0, 1, 0), 64), z[:64])


def test_bf16_rounding_is_single_rne():
    # float32 inputs: torch's float32 -> bfloat16 cast is one RNE rounding.
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(1 << 18) * 10.0).astype(np.float32)
    mine = s.round_to_bf16_bits(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)
    # exact midpoints between neighbours go to the even pattern, and values a
    # hair above a midpoint go up (a float32 detour would lose the hair).
    lo = np.float32(1.0)                                  # 0x3F80
    hi = np.float32(1.0078125)                            # 0x3F81
    mid = (float(lo) + float(hi)) / 2.0
    assert s.round_to_bf16_bits(np.array([mid]))[0] == 0x3F80
    assert s.round_to_bf16_bits(np.array([mid + 1e-12]))[0] == 0x3F81
    mid2 = (1.0078125 + 1.015625) / 2.0                   # between 0x3F81 and 0x3F82
    assert s.round_to_bf16_bits(np.array([mid2]))[0] == 0x3F82


def test_workload_shapes_and_distributions():
    w = s.workload("kontext_n8704")
    assert (w.B, w.H, w.N, w.d) == (1, 24, 8704, 128)
    q = s.head_fp64(w, 0, 5, "q")
    k = s.head_fp64(w, 0, 5, "k")
    v = s.head_fp64(w, 0, 5, "v")
    oc = s.outlier_channels(w.seed, 0, 5)
    assert len(set(oc.tolist())) == 4
    normal = np.setdiff1d(np.arange(128), oc)
    img = slice(w.n_text + w.n_ctx, w.N)
    ctx = slice(w.n_text, w.n_text + w.n_ctx)
    txt = slice(0, w.n_text)
    assert abs(q[img][:, normal].std() - 1.0) < 0.02
    assert abs(q[ctx][:, normal].std() - 1.5) < 0.03
    assert abs(q[txt][:, normal].std() - 3.0) < 0.1
    assert abs(q[img][:, oc].std() - 20.0) < 0.8
    assert abs(v[img][:, oc].std() - 1.0) < 0.1            # V has no outliers
    # K carries one offset per channel shared by all tokens
    off = k[img].mean(axis=0)
    assert abs((k[img] - off)[:, normal].std() - 1.0) < 0.02
    assert 1.0 < off[normal].std() < 3.0
    # config sizes
    assert [x.N for x in s.WORKLOADS] == [256, 1280, 4608, 8704, 16896]
    assert s.WORKLOADS[4].B == 2 and s.WORKLOADS[0].H == 2


def test_batch_elements_seeded_independently():
    w = s.workload("dit2048_cfg_n16896")
    a = s.normals(s.stream_key(w.seed, 0, 0, 0), 256)
    b = s.normals(s.stream_key(w.seed, 1, 0, 0), 256)
    assert not np.allclose(a, b)


def test_generate_deterministic():
    w = s.workload(0)
    g1 = s.generate(w)
    g2 = s.generate(w)
    for t in "qkv":
        assert s.sha256(g1[t]) == s.sha256(g2[t])
        assert g1[t].shape == (1, 2, 256, 128) and g1[t].dtype == np.uint16
