"""Host-side checks of the seeded workload generators and work counts."""
import torch

import workloads as W


def test_varlen_seqlens():
    w = W.WORKLOADS["fp16_varlen_t32768_h8_e64"]
    sl = W.workload_seqlens(w)
    assert sum(sl) == 32768
    assert all(8 <= n <= 4096 for n in sl[:-1]) and 1 <= sl[-1] <= 4096
    assert sl == W.varlen_seqlens(32768, 8, 4096, w.seed)  # deterministic
    cu = W.cu_seqlens_of(sl)
    assert cu[0] == 0 and cu[-1] == 32768 and all(a < b for a, b in zip(cu, cu[1:]))


def test_chunked_draws_regenerate_slices():
    shp = (3, 2, 5, 4)
    full = W.randn_chunked(shp, 7, torch.bfloat16)
    for i in range(3):
        assert torch.equal(full[i], W.randn_chunk(shp, 7, i, torch.bfloat16))
    assert not torch.equal(full[0], full[1])
    w = W.WORKLOADS["fp32_b1_h2_l64_e16"]
    q, k, v = W.make_inputs(w)
    assert q.dtype == torch.float32 and q.shape == (1, 2, 64, 16)
    assert torch.equal(q[0], W.make_slice(w, "q", 0)) and not torch.equal(q, k)


def test_work_counts():
    w2 = W.WORKLOADS["bf16_causal_b4_h16_l2048_e128"]
    assert W.flops(w2) == 4 * 16 * (2048 * 2049 // 2) * 512  # 6.875e10
    w4 = W.WORKLOADS["bf16_gqa_decode_b64_hq32_hkv8_s16384_e128"]
    assert W.kv_bytes(w4) == 64 * 8 * 16384 * 256 * 2  # 4.295e9
    w5 = W.WORKLOADS["fp16_causal_b1_h64_l2048_e96"]
    assert abs(W.flops(w5) - 5.16e10) / 5.16e10 < 0.01
    w1 = W.WORKLOADS["fp32_b1_h2_l64_e16"]
    assert W.flops(w1) == 2 * 64 * 64 * 64
    w3 = W.WORKLOADS["fp16_varlen_t32768_h8_e64"]
    f3 = W.flops(w3)
    assert 5e10 < f3 < 2e11
