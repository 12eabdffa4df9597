// quantize.cuh -- BF16 Q/K/V -> E4M3 codes with one FP32 absmax scale per
// (batch, head, 64-token block), K smoothed by its per-channel mean.
//
// Scheme: FP8 scaled dot-product attention with Q, K and V quantized ("NVIDIA
// RTX AI optimiert FLUX.1 fuer Bilddaten mit niedriger Genauigkeit", SDPA
// quantization paragraph; SageAttention named there as the lineage).  The
// pages fix no granularity, order or rounding; this file follows these
// readings, bit for bit:
//   mu[c]  = (sum over 64-token blocks j ascending of
//             (sum over the block's tokens ascending of k[n][c])) / N,
//            every sum a sequential binary32 sum from +0, one RN division;
//   x      = q, fl32(k - mu[c]) or v;
//   amax   = max |x| over the block's 64 x 128 values;
//   s      = amax / 448, inv = 448 / amax (RN divisions; 0 and 0 if amax = 0);
//   code   = E4M3_RNE_satfinite(fl32(x * inv));
//   sv_max = max over the head's V block scales.
// All three kernels read BF16 [B,H,N,128] and write codes in the same layout.
#pragma once

#include "device.cuh"

namespace fqa {

// Level 1 of the K mean: partial[b,h,j,c] = sequential sum of the block's 64
// tokens of channel c.  grid (N/64, H, B), 128 threads (one per channel).
__global__ void __launch_bounds__(128) kmean_partial_kernel(const __nv_bfloat16* __restrict__ k,
                                                            float* __restrict__ partial, int H,
                                                            int N) {
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z, c = threadIdx.x;
  const size_t head = (size_t)b * H + h;
  const __nv_bfloat16* src = k + (head * N + (size_t)j * kQBlock) * kHeadDim + c;
  float v[kQBlock];
#pragma unroll
  for (int n = 0; n < kQBlock; ++n) v[n] = __bfloat162float(src[(size_t)n * kHeadDim]);
  float p = 0.0f;
#pragma unroll
  for (int n = 0; n < kQBlock; ++n) p = __fadd_rn(p, v[n]);
  partial[(head * (N / kQBlock) + j) * kHeadDim + c] = p;
}

// Level 2: mu = (sequential sum of the partials over blocks) / N; also
// clears sv_max for the quantize kernel's atomic maximum.
// grid (B*H), 128 threads.
__global__ void __launch_bounds__(128) kmean_reduce_kernel(const float* __restrict__ partial,
                                                           float* __restrict__ k_mean,
                                                           float* __restrict__ sv_max, int N) {
  const size_t head = blockIdx.x;
  const int c = threadIdx.x, nblk = N / kQBlock;
  const float* src = partial + head * nblk * kHeadDim + c;
  float t = 0.0f;
  for (int j = 0; j < nblk; ++j) t = __fadd_rn(t, src[(size_t)j * kHeadDim]);
  k_mean[head * kHeadDim + c] = __fdiv_rn(t, (float)N);
  if (c == 0) sv_max[head] = 0.0f;
}

__device__ __forceinline__ float block_max_256(float v, float* red, int slot) {
  // max over the 256 threads of the CTA; red holds 8 floats for this slot
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[slot * 8 + (threadIdx.x >> 5)] = v;
  return v;
}

// One CTA quantizes one 64-token block of Q, K and V for one (b, h).
// Thread t owns token row t/4 and channels [32*(t%4), 32*(t%4)+32).
// grid (N/64, H, B), 256 threads.
__global__ void __launch_bounds__(256) quantize_qkv_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const float* __restrict__ k_mean,
    uint8_t* __restrict__ q8, uint8_t* __restrict__ k8, uint8_t* __restrict__ v8,
    float* __restrict__ sq, float* __restrict__ sk, float* __restrict__ sv,
    float* __restrict__ sv_max, int H, int N) {
  __shared__ float red[3 * 8];
  __shared__ float mu[kHeadDim];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x, row = t >> 2, c0 = (t & 3) * 32;
  const size_t head = (size_t)b * H + h;
  const size_t elem0 = (head * N + (size_t)j * kQBlock + row) * kHeadDim + c0;

  // issue all global loads first: 3 tensors x 64 bytes per thread
  uint4 raw[3][4];
  const uint4* srcq = reinterpret_cast<const uint4*>(q + elem0);
  const uint4* srck = reinterpret_cast<const uint4*>(k + elem0);
  const uint4* srcv = reinterpret_cast<const uint4*>(v + elem0);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    raw[0][i] = __ldg(srcq + i);
    raw[1][i] = __ldg(srck + i);
    raw[2][i] = __ldg(srcv + i);
  }
  if (t < kHeadDim) mu[t] = k_mean[head * kHeadDim + t];
  __syncthreads();

  float x[3][32];
#pragma unroll
  for (int s = 0; s < 3; ++s) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[s][i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(h2[e]);
        x[s][i * 8 + 2 * e] = f.x;
        x[s][i * 8 + 2 * e + 1] = f.y;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) x[1][i] = __fsub_rn(x[1][i], mu[c0 + i]);

  float amax[3];
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(x[s][i]));
    block_max_256(m, red, s);
  }
  __syncthreads();
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    float m = red[s * 8];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red[s * 8 + w]);
    amax[s] = m;
  }

  uint8_t* dst[3] = {q8, k8, v8};
  float* scl[3] = {sq, sk, sv};
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    const float a = amax[s];
    const float scale = a > 0.0f ? __fdiv_rn(a, 448.0f) : 0.0f;
    const float inv = a > 0.0f ? __fdiv_rn(448.0f, a) : 0.0f;
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t lo = e4m3x2(__fmul_rn(x[s][4 * i], inv), __fmul_rn(x[s][4 * i + 1], inv));
      uint32_t hi = e4m3x2(__fmul_rn(x[s][4 * i + 2], inv), __fmul_rn(x[s][4 * i + 3], inv));
      w[i] = lo | (hi << 16);
    }
    uint4* o = reinterpret_cast<uint4*>(dst[s] + elem0);
    o[0] = make_uint4(w[0], w[1], w[2], w[3]);
    o[1] = make_uint4(w[4], w[5], w[6], w[7]);
    if (t == 0) {
      scl[s][head * (N / kQBlock) + j] = scale;
      if (s == 2) atomicMax(reinterpret_cast<unsigned int*>(sv_max + head), __float_as_uint(scale));
    }
  }
}

// Standalone conversion kernel: every binary32 input -> its E4M3 code via the
// same instruction the quantizer uses (for exhaustive codec checks).
__global__ void e4m3_encode_kernel(const float* __restrict__ x, uint8_t* __restrict__ out, size_t n) {
  size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 2;
  const size_t stride = (size_t)gridDim.x * blockDim.x * 2;
  for (; i + 1 < n; i += stride) {
    uint32_t c = e4m3x2(x[i], x[i + 1]);
    out[i] = (uint8_t)(c & 0xFF);
    out[i + 1] = (uint8_t)(c >> 8);
  }
  if (i < n) out[i] = (uint8_t)(e4m3x2(x[i], 0.0f) & 0xFF);
}

}  // namespace fqa
