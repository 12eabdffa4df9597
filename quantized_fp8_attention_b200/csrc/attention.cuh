// attention.cuh -- definitions shared by the attention kernels (the kernel
// itself, persistent and two Q tiles per CTA, is in attention_ws.cuh).
//
// FP8 path: scaled dot-product attention with Q, K, V quantized to E4M3 and
// the attention itself kept in FP8 ("NVIDIA RTX AI optimiert FLUX.1 fuer
// Bilddaten mit niedriger Genauigkeit", SDPA quantization and Table-1
// paragraphs; "NVIDIA RTX AI, 저정밀 양자화로 FLUX.1 Kontext 최적화", SDPA
// paragraph).  BF16 path: the unquantized comparison backend ("FLUX 3 Image
// Klein Base", section "왜 이런 차이가 나나": VANILLA BF16 attention, about
// 60% of DiT kernel time on B200).
//
// Per query row i (64-token block I) and KV tile t of 128 keys, ascending:
//   x_j  = (q8_i . k8_j) * sq_I * sk_J * scale * log2(e)      (J = j / 64)
//   m_t  = max(m_{t-1}, max_j x_j)        exact running max, every tile
//   p_j  = 2^(x_j - m_t);  l = l * 2^(m_{t-1} - m_t) + sum_j p_j
//   P_j  = E4M3(p_j * 448 * sv_J / sv_max)
//   O    = O * 2^(m_{t-1} - m_t) + P . v8     (tensor cores, FP32 in TMEM)
// and at the end out = O * (sv_max / 448) / l.  The BF16 path drops the
// scales, keeps P in BF16 and ends with out = O / l.
// Shared memory: Q, K and V tiles 128 rows x 128 B, 128-byte swizzle (TMA
// writes it, the MMA descriptors read it).  Q and K are K-major operands;
// V tiles stay token-major and feed the P.V MMA as an MN-major B operand.
#pragma once

#include "device.cuh"

namespace fqa {

constexpr int kBlockM = 128;   // query rows per CTA
constexpr int kBlockN = 128;   // keys per KV tile (part of the FP8 rounding rule)
constexpr int kMaxScaleBlocks = 1024;   // N <= 65536

// p for two keys at once: 2^(x - m) with x = fl(S * a) already rounded and
// m = max x.  x - m is exact near the maximum (Sterbenz), so the row maximum
// gets p = 1 exactly and the row sum l carries no common rounding factor (a
// fused S * a - m would give the maximum p = 2^delta, delta the rounding
// residue of m, and bias l by ~|m| 2^-24).  The subtraction is written as
// fma(x, 1, -m) so that the multiply producing x can never be fused into it.
__device__ __forceinline__ float2 exp2_pair(float2 x, float2 nm2) {
  const float2 d = f2_fma(x, make_float2(1.0f, 1.0f), nm2);
  return make_float2(ex2_approx(d.x), ex2_approx(d.y));
}

struct AttnParams {
  int B, H, N;
  float softmax_scale;
  const float* sq;      // [B,H,N/64]   (FP8 path only)
  const float* sk;
  const float* sv;
  const float* sv_max;  // [B,H]
  void* out;            // [B,H,N,128] BF16 or FP32
  int out_f32;
  uint32_t* status;     // device status word
  const uint8_t* q8 = nullptr;       // FP8: the code tensors (read by the short-tile correction)
  const uint8_t* k8 = nullptr;
  const uint32_t* kmask = nullptr;   // FP8, key-masked kernel: excluded keys [B,H,ceil(N/32)]
  float2* row_stats = nullptr;       // FP8, key-masked kernel: (m, l) per row [B,H,N]
  int out_P = 1;                     // FP8: > 1 writes out in the sequence all-to-all layout
  int patch = 0;                     // FP8 with kmask: apply it by patching K / V tiles (see attention_fp8.cuh)
};

__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

}  // namespace fqa
