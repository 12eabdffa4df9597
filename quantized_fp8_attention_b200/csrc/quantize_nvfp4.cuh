// quantize_nvfp4.cuh -- Q and smoothed K in NVFP4 for the FP4 Q.K variant:
// E2M1 elements with one unsigned E4M3 scale per 16 channels, under the FP8
// path's per-(b, h, 64-token block) FP32 scale ("NVIDIA RTX AI optimiert
// FLUX.1 fuer Bilddaten mit niedriger Genauigkeit", SDPA quantization
// paragraph: the FP8 and FP4 schemes differ only in the precision of the Q,
// K, V projections; attention stays in FP8).  The readings, bit for bit:
//   s1  = fl32(amax / 2688)                (6 * 448: group scales up to 448)
//   per token and 16-channel group: t = fl32(amax_g / fl32(s1 * 6)),
//   s2  = E4M3_RNE_satfinite(t),  dg = fl32(s1 * dec(s2)),
//   code = E2M1_RNE_satfinite(fl32(x / dg))   (0 where dg == 0)
// amax == 0 (or s1 underflowing to 0) flushes the block: s1 = 0, scales and
// codes 0.  x = q, or fl32(k - k_mean) for K (k_mean from fqa_quantize).
// One CTA per (tensor, b, h, 64-token block); thread t handles the 16-byte
// chunks t, t+256, t+512, t+768 of the block (8 channels each: a 16-channel
// group is the chunk pair of threads 2i, 2i+1).
#pragma once

#include "device.cuh"

namespace fqa {

constexpr int kNv4Threads = 256;

__global__ void __launch_bounds__(kNv4Threads) quantize_nvfp4_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const float* __restrict__ k_mean, uint8_t* __restrict__ q4, uint8_t* __restrict__ k4,
    uint8_t* __restrict__ sfq, uint8_t* __restrict__ sfk, float* __restrict__ sq1,
    float* __restrict__ sk1, int B, int H, int N) {
  const int nblk = (N + 63) / 64;
  const int units = B * H * nblk;
  const int u = blockIdx.x % units;
  const bool is_k = blockIdx.x >= units;
  const int hd = u / nblk, j = u - hd * nblk;
  const int rows = min(64, N - 64 * j);
  const size_t row0 = (size_t)hd * N + 64 * j;
  const __nv_bfloat16* src = (is_k ? k : q) + row0 * kHeadDim;
  const int t = threadIdx.x;
  __shared__ float red[kNv4Threads / 32];

  float x[4][8];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = t + kNv4Threads * i;       // chunk: token c / 16, channels 8 (c % 16) ..
    const int tok = c >> 4, ch0 = (c & 15) * 8;
    if (tok < rows) {
      const uint4 raw = *reinterpret_cast<const uint4*>(src + (size_t)tok * kHeadDim + ch0);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        x[i][2 * e] = f.x;
        x[i][2 * e + 1] = f.y;
      }
      if (is_k) {
        const float* mu = k_mean + (size_t)hd * kHeadDim + ch0;
#pragma unroll
        for (int e = 0; e < 8; ++e) x[i][e] = __fsub_rn(x[i][e], __ldg(mu + e));
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[i][e] = 0.0f;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[i][e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((t & 31) == 0) red[t >> 5] = amax;
  __syncthreads();
  float a = red[0];
#pragma unroll
  for (int w = 1; w < kNv4Threads / 32; ++w) a = fmaxf(a, red[w]);
  const float s1 = a > 0.0f ? __fdiv_rn(a, 2688.0f) : 0.0f;
  const float den = __fmul_rn(s1, 6.0f);
  uint8_t* codes = (is_k ? k4 : q4) + row0 * (kHeadDim / 2);
  uint8_t* sf = (is_k ? sfk : sfq) + row0 * (kHeadDim / 16);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = t + kNv4Threads * i;
    const int tok = c >> 4;
    float ag = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ag = fmaxf(ag, fabsf(x[i][e]));
    ag = fmaxf(ag, __shfl_xor_sync(0xffffffffu, ag, 1));          // the group's other chunk
    uint32_t s2 = 0;
    float dg = 0.0f;
    if (s1 > 0.0f) {
      s2 = e4m3x2(__fdiv_rn(ag, den), 0.0f) & 0xFFu;
      dg = __fmul_rn(s1, e4m3x2_to_f2(s2).x);
    }
    uint32_t w = 0;
    if (dg > 0.0f) {
#pragma unroll
      for (int e = 0; e < 8; e += 2)
        w |= e2m1x2(__fdiv_rn(x[i][e], dg), __fdiv_rn(x[i][e + 1], dg)) << (4 * e);
    }
    if (tok < rows) {
      *reinterpret_cast<uint32_t*>(codes + (size_t)c * 4) = w;     // 8 codes of 4 bits
      if ((c & 1) == 0) sf[c >> 1] = (uint8_t)s2;                  // one scale per 16 channels
    }
  }
  if (t == 0) (is_k ? sk1 : sq1)[u] = s1;
}

// Standalone E2M1 conversion (for exhaustive codec checks): out[i] holds
// the code of x[2i] in bits [0,4) and of x[2i+1] in bits [4,8).
__global__ void e2m1_encode_kernel(const float* __restrict__ x, uint8_t* __restrict__ out, size_t npairs) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < npairs; i += (size_t)gridDim.x * blockDim.x)
    out[i] = (uint8_t)e2m1x2(x[2 * i], x[2 * i + 1]);
}

}  // namespace fqa
