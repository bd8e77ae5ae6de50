"""GPU parity of the layer glue: f1 = SiLU(x W1 + b1) -> [U | V | Q | K],
f2 = y W2 + b2, and one whole layer (f1 -> attention -> f2), each against the
fp64 oracle on the same bf16-rounded inputs."""
import numpy as np
import pytest
import torch

import generative_recommender_attention_jagged_b200 as hstu
import oracle
import synth
from oracle import layer as olayer

from .gpu_helpers import BF16_TOL, F32_TOL, dev, host64, rel_err, sample_rows

pytestmark = pytest.mark.gpu

H, D, DM = 4, 128, 512


def weights(seed: int, dtype=torch.bfloat16, bias_std: float = 0.05):
    rng = np.random.default_rng([77, seed])
    w = synth.layer_weights(rng, DM, H, D)
    # nonzero biases so that the epilogue bias is exercised (the workloads use zero)
    b1 = (rng.standard_normal(4 * H * D) * bias_std).astype(np.float32)
    b2 = (rng.standard_normal(DM) * bias_std).astype(np.float32)
    w1 = torch.from_numpy(w.w1).to(dtype)
    w2 = torch.from_numpy(w.w2).to(dtype)
    return w1, b1, w2, b2


def x_rows(T: int, seed: int, dtype=torch.bfloat16):
    rng = np.random.default_rng([78, seed])
    return synth.draw_normal(rng, (T, DM), 1.0, dtype)


@pytest.mark.parametrize("T", [1, 37, 640, 1001])
def test_f1_matches_oracle(T):
    w1, b1, _, _ = weights(T)
    x = x_rows(T, T)
    z = hstu.hstu_layer_f1(dev(x), dev(w1), dev(b1))
    torch.cuda.synchronize()
    u, v, q, k = olayer.f1(host64(x), host64(w1), b1, H, D)
    want = np.concatenate([u, v.reshape(T, -1), q.reshape(T, -1), k.reshape(T, -1)], axis=1)
    assert rel_err(host64(z), want) <= BF16_TOL
    # the block order [U | V | Q | K], head-major inside, through the split views
    gu, gv, gq, gk = hstu.split_uvqk(z, H, D)
    assert rel_err(host64(gq), q) <= BF16_TOL
    assert rel_err(host64(gk), k) <= BF16_TOL
    assert rel_err(host64(gv), v) <= BF16_TOL
    assert rel_err(host64(gu), u) <= BF16_TOL


@pytest.mark.parametrize("T", [5, 700])
def test_f2_matches_oracle(T):
    _, _, w2, b2 = weights(T + 1)
    rng = np.random.default_rng([79, T])
    y = synth.draw_normal(rng, (T, H * D), 1.0, torch.bfloat16)
    out = hstu.hstu_layer_f2(dev(y), dev(w2), dev(b2))
    torch.cuda.synchronize()
    assert rel_err(host64(out), olayer.f2(host64(y), host64(w2), b2)) <= BF16_TOL


def test_linear_without_bias_and_with_strided_rows():
    T = 300
    w1, _, _, _ = weights(3)
    x_wide = x_rows(T, 3).repeat(1, 2)          # [T, 1024]: use the first 512 columns (row stride 1024)
    x = dev(x_wide)[:, :DM]
    out_wide = torch.zeros(T, 4 * H * D + 64, dtype=torch.bfloat16, device="cuda")
    out = out_wide[:, :4 * H * D]
    hstu.hstu_linear(x, dev(w1), None, silu=True, out=out)
    torch.cuda.synchronize()
    u, v, q, k = olayer.f1(host64(x_wide)[:, :DM], host64(w1), np.zeros(4 * H * D), H, D)
    want = np.concatenate([u, v.reshape(T, -1), q.reshape(T, -1), k.reshape(T, -1)], axis=1)
    assert rel_err(host64(out), want) <= BF16_TOL
    assert torch.count_nonzero(out_wide[:, 4 * H * D:]) == 0   # nothing written past the row


def test_linear_fp32():
    T = 200
    w1, b1, _, _ = weights(9, torch.float32)
    x = x_rows(T, 9, torch.float32)
    z = hstu.hstu_layer_f1(dev(x), dev(w1), dev(b1))
    torch.cuda.synchronize()
    u, v, q, k = olayer.f1(host64(x), host64(w1), b1, H, D)
    want = np.concatenate([u, v.reshape(T, -1), q.reshape(T, -1), k.reshape(T, -1)], axis=1)
    assert rel_err(host64(z), want) <= F32_TOL


def test_whole_layer_matches_oracle():
    """x -> f1 -> attention on f1's strided u/v/q/k views -> f2, sampled rows."""
    s = synth.workload_stack("layer_bf16", num_layers=1)
    rab_pos, rab_ts, w = s.layers[0]
    w1 = torch.from_numpy(w.w1).to(torch.bfloat16)
    w2 = torch.from_numpy(w.w2).to(torch.bfloat16)
    x = dev(s.x)
    z = hstu.hstu_layer_f1(x, dev(w1), dev(w.b1))
    u, v, q, k = hstu.split_uvqk(z, H, D)
    y = hstu.hstu_attn_fwd(q, k, v, u, dev(s.seq_offsets, torch.int32), dev(s.timestamps, torch.int64),
                           dev(rab_pos, torch.float32), dev(rab_ts, torch.float32), n_max=s.n_max,
                           alpha=s.alpha, max_seq_len=s.n_max)
    x_next = hstu.hstu_layer_f2(y, dev(w2), dev(w.b2))
    torch.cuda.synchronize()
    got = host64(x_next)
    assert np.isfinite(got).all()
    rows = sample_rows(s.seq_offsets, None, per_user=2)
    want = olayer.layer(host64(s.x), host64(w1), w.b1, host64(w2), w.b2, s.seq_offsets, s.timestamps, None,
                        rab_pos, rab_ts, s.alpha, s.n_max, H, D, rows=rows)
    assert rel_err(got[rows], want) <= BF16_TOL


@pytest.mark.parametrize("T", [1, 300, 4099])
def test_own_gemm_and_cublas_agree_with_the_oracle(T):
    """bf16 f1 runs the library's SM-pair tcgen05 GEMM (bias and SiLU in its
    epilogue), f2 (512 columns) cuBLASLt; both routes must agree with the
    oracle within the bf16 tolerance."""
    w1, b1, w2, b2 = weights(T + 7)
    x = dev(x_rows(T, T + 7))
    z_own = hstu.hstu_layer_f1(x, dev(w1), dev(b1))
    z_lib = hstu.hstu_layer_f1(x, dev(w1), dev(b1), force_cublas=True)
    y_own = hstu.hstu_layer_f2(z_own[:, :DM].contiguous(), dev(w2), dev(b2))
    y_lib = hstu.hstu_layer_f2(z_own[:, :DM].contiguous(), dev(w2), dev(b2), force_cublas=True)
    torch.cuda.synchronize()
    u, v, q, k = olayer.f1(host64(x), host64(w1), b1, H, D)
    want = np.concatenate([u, v.reshape(T, -1), q.reshape(T, -1), k.reshape(T, -1)], axis=1)
    assert rel_err(host64(z_own), want) <= BF16_TOL
    assert rel_err(host64(z_lib), want) <= BF16_TOL
    y_want = olayer.f2(host64(z_own[:, :DM]), host64(w2), b2)
    assert rel_err(host64(y_own), y_want) <= BF16_TOL
    assert rel_err(host64(y_lib), y_want) <= BF16_TOL
    assert not torch.equal(z_own, z_lib) or T == 1   # two different kernels ran


def test_own_gemm_plain_wide_output():
    T = 777
    w1, b1, _, _ = weights(21)
    x = dev(x_rows(T, 21))
    own = hstu.hstu_linear(x, dev(w1), dev(b1))               # 2048 columns, no activation
    lib = hstu.hstu_linear(x, dev(w1), dev(b1), force_cublas=True)
    torch.cuda.synchronize()
    want = host64(x) @ host64(w1) + b1
    assert rel_err(host64(own), want) <= BF16_TOL and rel_err(host64(lib), want) <= BF16_TOL
    assert not torch.equal(own, lib)


@pytest.mark.parametrize("K,N,silu", [(1024, 1024, True), (1024, 2048, False), (576, 384, True)])
def test_own_gemm_long_k_schedule(K, N, silu):
    """Shapes other than the layer's: K = 1024 (16 K-blocks through the 6-stage
    ring) runs the library's GEMM, a 384-column output (not a multiple of the
    256-column pair tile) goes to cuBLASLt + the SiLU pass."""
    T = 1000
    rng = np.random.default_rng(K + N)
    x = torch.from_numpy(rng.normal(size=(T, K)).astype(np.float32)).to(torch.bfloat16).cuda()
    w = torch.from_numpy(rng.uniform(-0.05, 0.05, size=(K, N)).astype(np.float32)).to(torch.bfloat16).cuda()
    b = torch.from_numpy(rng.normal(0, 0.1, size=N).astype(np.float32)).cuda()
    got = hstu.hstu_linear(x, w, b, silu=silu)
    torch.cuda.synchronize()
    z = host64(x) @ host64(w) + host64(b)
    want = olayer.silu(z) if silu else z
    assert rel_err(host64(got), want) <= BF16_TOL
