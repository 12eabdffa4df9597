// attention.cuh -- non-causal attention forward on tcgen05 tensor cores.
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
//
// CTA = one (b, h, 128-row Q tile); 192 threads:
//   warps 0-3  softmax + O correction + epilogue (thread = query row = TMEM lane)
//   warp 4     TMA producer (Q once; K and V tiles through a kStages ring)
//   warp 5     TMEM allocator and single-thread tcgen05.mma issuer
// TMEM (256 columns): S at [0,128), O at [128,256); P overwrites the top of S
// (FP8: 32 columns at 96, 4 codes per column; BF16: 64 columns at 64) once the
// softmax threads hold S in registers.  The next S = Q K^T is issued after
// the P.V MMA that reads P; tcgen05.mma operations from one thread execute in
// issue order, so the overwrite cannot overtake the read.
// Shared memory: Q, K and V tiles 128 rows x 128 B, 128-byte swizzle (TMA
// writes it, the MMA descriptors read it).  Q and K are K-major operands;
// V tiles stay token-major and feed the P.V MMA as an MN-major B operand.
#pragma once

#include "device.cuh"

namespace fqa {

constexpr int kBlockM = 128;   // query rows per CTA
constexpr int kBlockN = 128;   // keys per KV tile (part of the FP8 rounding rule)
constexpr int kAttnThreads = 192;
constexpr int kMaxScaleBlocks = 1024;   // N <= 65536

// Of every 8 exponentials (pairs of keys) this many are evaluated by the FMA
// pipe polynomial instead of the MUFU ex2 unit, to balance the two pipes.
#ifndef FQA_EXP2_POLY_PER8
#define FQA_EXP2_POLY_PER8 0
#endif
constexpr int kPolyPer8 = FQA_EXP2_POLY_PER8;

// p for two keys at once: 2^(x - m) with x = fl(S * a) already rounded and
// m = max x.  x - m is exact near the maximum (Sterbenz), so the row maximum
// gets p = 1 exactly and the row sum l carries no common rounding factor (a
// fused S * a - m would give the maximum p = 2^delta, delta the rounding
// residue of m, and bias l by ~|m| 2^-24).  The subtraction is written as
// fma(x, 1, -m) so that the multiply producing x can never be fused into it.
template <bool kPoly>
__device__ __forceinline__ float2 exp2_pair(float2 x, float2 nm2) {
  const float2 d = f2_fma(x, make_float2(1.0f, 1.0f), nm2);
  if constexpr (kPoly) return exp2_poly2(d);
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
};

template <bool kFP8>
struct AttnTraits {
  static constexpr int kElt = kFP8 ? 1 : 2;
  static constexpr int kTileBytes = kBlockM * kHeadDim * kElt;      // one 128 x 128 tile
  static constexpr int kStages = 2;
  static constexpr int kKStep = kFP8 ? 32 : 16;                     // MMA K per instruction
  static constexpr int kSteps = 128 / kKStep;                       // MMAs per 128-wide K
  static constexpr uint32_t kFmt = kFP8 ? 0u : 1u;                  // E4M3 / BF16
  static constexpr uint32_t kPCol = kFP8 ? 96u : 64u;               // P columns inside S
  static constexpr uint32_t kIdescS = make_idesc(kFmt, kFmt, 128, 128, 0);
  static constexpr uint32_t kIdescPV = make_idesc(kFmt, kFmt, 128, 128, 1);
  // shared-memory carve-up (offsets from a 1024-aligned base)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  static constexpr int kNumBars = 3 * kStages + 4;
  static constexpr int kOffScale = kOffBar + 8 * kNumBars + 16;
  static constexpr int kScaleBytes = kFP8 ? 2 * kMaxScaleBlocks * 4 : 0;
  static constexpr int kSmemBytes = kOffScale + kScaleBytes + 1024;  // + alignment slack
};

// Descriptor of K-step `k` of a 128-row, K-major, 128-byte-swizzled tile.
// FP8 rows are exactly 128 B; BF16 tiles are two 64-column halves 16 KB apart.
template <bool kFP8>
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int k) {
  uint32_t off = kFP8 ? (uint32_t)k * 32u : (uint32_t)(k >> 2) * 16384u + (uint32_t)(k & 3) * 32u;
  return make_sdesc_sw128(tile + off, 16, 1024);
}
// Descriptor of K-step `k` (keys) of a token-major V tile used MN-major:
// 8-key groups 1024 B apart; BF16 d-halves (MN chunks) 16 KB apart.
template <bool kFP8>
__device__ __forceinline__ uint64_t desc_v(uint32_t tile, int k) {
  uint32_t off = (uint32_t)k * (uint32_t)AttnTraits<kFP8>::kKStep * 128u;
  return make_sdesc_sw128(tile + off, 16384, 1024);
}

__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

template <bool kFP8>
__global__ void __launch_bounds__(kAttnThreads, kFP8 ? 2 : 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using T = AttnTraits<kFP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + T::kOffQ;
  uint8_t* sK = smem + T::kOffK;
  uint8_t* sV = smem + T::kOffV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::kOffBar);
  uint64_t* fullK = bars;                       // [kStages]
  uint64_t* fullV = bars + T::kStages;          // [kStages]
  uint64_t* empty = bars + 2 * T::kStages;      // [kStages]
  uint64_t* barQ = bars + 3 * T::kStages;
  uint64_t* barS = barQ + 1;
  uint64_t* barP = barQ + 2;
  uint64_t* barO = barQ + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* skc = reinterpret_cast<float*>(smem + T::kOffScale);   // sk_J * scale * log2 e
  float* pvc = skc + kMaxScaleBlocks;                            // 448 * sv_J / sv_max

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int N = p.N, nkv = N / kBlockN, nblk = N / 64;
  const size_t head = (size_t)b * p.H + h;
  const int row0 = (int)(head * N) + qt * kBlockM;     // first global row of this Q tile
  const int kv_row0 = (int)(head * N);
  const float c_log2e = p.softmax_scale * 1.4426950408889634f;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::kStages; ++s) {
      mbar_init(&fullK[s], 1);
      mbar_init(&fullV[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(barQ, 1);
    mbar_init(barS, 1);
    mbar_init(barP, kBlockM);
    mbar_init(barO, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  float svmax = 0.0f;
  if constexpr (kFP8) {
    svmax = p.sv_max[head];
    for (int j = threadIdx.x; j < nblk; j += kAttnThreads) {
      skc[j] = p.sk[head * nblk + j] * c_log2e;
      pvc[j] = svmax > 0.0f ? 448.0f * (p.sv[head * nblk + j] / svmax) : 0.0f;
    }
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp == 4) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(barQ, T::kTileBytes);
      if constexpr (kFP8) {
        tma_load_2d(sQ, &tmQ, barQ, 0, row0);
      } else {
        tma_load_2d(sQ, &tmQ, barQ, 0, row0);
        tma_load_2d(sQ + 16384, &tmQ, barQ, 64, row0);
      }
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int s = j % T::kStages, r = j / T::kStages;
        if (!mbar_wait(&empty[s], (r & 1) ^ 1, abort_flag, p.status)) break;
        const int y = kv_row0 + j * kBlockN;
        mbar_arrive_expect_tx(&fullK[s], T::kTileBytes);
        mbar_arrive_expect_tx(&fullV[s], T::kTileBytes);
        if constexpr (kFP8) {
          tma_load_2d(sK + s * T::kTileBytes, &tmK, &fullK[s], 0, y);
          tma_load_2d(sV + s * T::kTileBytes, &tmV, &fullV[s], 0, y);
        } else {
          tma_load_2d(sK + s * T::kTileBytes, &tmK, &fullK[s], 0, y);
          tma_load_2d(sK + s * T::kTileBytes + 16384, &tmK, &fullK[s], 64, y);
          tma_load_2d(sV + s * T::kTileBytes, &tmV, &fullV[s], 0, y);
          tma_load_2d(sV + s * T::kTileBytes + 16384, &tmV, &fullV[s], 64, y);
        }
        issued = j + 1;
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA exits
        mbar_wait_drain(barQ, 0);
        for (int j = (issued > T::kStages ? issued - T::kStages : 0); j < issued; ++j) {
          const int s = j % T::kStages, r = j / T::kStages;
          mbar_wait_drain(&fullK[s], r & 1);
          mbar_wait_drain(&fullV[s], r & 1);
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t aQ = smem_u32(sQ);
      bool ok = mbar_wait(barQ, 0, abort_flag, p.status);
      for (int j = 0; ok && j < nkv; ++j) {
        const int s = j % T::kStages, r = j / T::kStages;
        const uint32_t aK = smem_u32(sK + s * T::kTileBytes);
        const uint32_t aV = smem_u32(sV + s * T::kTileBytes);
        if (!(ok = mbar_wait(&fullK[s], r & 1, abort_flag, p.status))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < T::kSteps; ++k) {
          if constexpr (kFP8)
            mma_f8_ss(tS, desc_kmajor<true>(aQ, k), desc_kmajor<true>(aK, k), T::kIdescS, k > 0);
          else
            mma_bf16_ss(tS, desc_kmajor<false>(aQ, k), desc_kmajor<false>(aK, k), T::kIdescS,
                        k > 0);
        }
        tc_commit(barS);
        if (!(ok = mbar_wait(barP, j & 1, abort_flag, p.status))) break;
        if (!(ok = mbar_wait(&fullV[s], r & 1, abort_flag, p.status))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < T::kSteps; ++k) {
          const uint32_t aP = tS + T::kPCol + 8u * (uint32_t)k;
          if constexpr (kFP8)
            mma_f8_ts(tO, aP, desc_v<true>(aV, k), T::kIdescPV, (j > 0 || k > 0));
          else
            mma_bf16_ts(tO, aP, desc_v<false>(aV, k), T::kIdescPV, (j > 0 || k > 0));
        }
        tc_commit(&empty[s]);
      }
      tc_commit(barO);     // fires when every MMA above has completed
      if (!ok) mbar_wait_drain(barO, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax warpgroup
    const int r = threadIdx.x;                       // row in tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float a_row = 0.0f;
    if constexpr (kFP8) a_row = p.sq[head * nblk + (qt * kBlockM + r) / 64];
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      // warp-uniform exit: the TMEM accesses below are .sync.aligned
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(barS, j & 1, abort_flag, p.status)))) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + lane_off + 32u * c, sr[c]);
      tmem_wait_ld();
      // scores in log2 units, rounded once: x = fl(S * a) (per 64-key block scale)
      float a0, a1;
      if constexpr (kFP8) {
        a0 = a_row * skc[2 * j];
        a1 = a_row * skc[2 * j + 1];
      } else {
        a0 = a1 = c_log2e;
      }
      float2 X[64];
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        const float a = (e < 32) ? a0 : a1;
        X[e] = f2_mul(make_float2(__uint_as_float(sr[e >> 4][(2 * e) & 31]),
                                  __uint_as_float(sr[e >> 4][(2 * e + 1) & 31])),
                      make_float2(a, a));
      }
      // tile max of x: 4 independent chains of 3-input maxima over 16 pairs each
      float cm[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        cm[r] = fmaxf(X[16 * r].x, X[16 * r].y);
#pragma unroll
        for (int t = 1; t < 16; ++t) cm[r] = fmax3(cm[r], X[16 * r + t].x, X[16 * r + t].y);
      }
      const float tmax = fmaxf(fmax3(cm[0], cm[1], cm[2]), cm[3]);
      const float m_new = fmaxf(m, tmax);
      const float alpha = ex2_approx(m - m_new);     // 0 on the first tile
      // O correction: rescale the accumulated rows whose max moved.  The
      // barS phase we waited on completes after the previous P.V MMA.
      if (j > 0 && __any_sync(0xffffffffu, m_new != m)) {
        const float2 al2 = make_float2(alpha, alpha);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + 32u * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float2 v = f2_mul(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), al2);
            o[e] = __float_as_uint(v.x);
            o[e + 1] = __float_as_uint(v.y);
          }
          tmem_st32(tO + lane_off + 32u * c, o);
        }
      }
      const float2 nm2 = make_float2(-m_new, -m_new);
      float2 l2 = make_float2(0.0f, 0.0f);
      if constexpr (kFP8) {
        uint32_t pw[32];
#pragma unroll
        const float c0 = pvc[2 * j], c1 = pvc[2 * j + 1];
#pragma unroll
        for (int w = 0; w < 32; ++w) {
          const float cc = (w < 16) ? c0 : c1;
          const float2 c2 = make_float2(cc, cc);
          float2 p01, p23;
          if ((w % 4) < kPolyPer8 / 2) {
            p01 = exp2_pair<true>(X[2 * w], nm2);
            p23 = exp2_pair<true>(X[2 * w + 1], nm2);
          } else if ((w % 4) == kPolyPer8 / 2 && (kPolyPer8 & 1)) {
            p01 = exp2_pair<true>(X[2 * w], nm2);
            p23 = exp2_pair<false>(X[2 * w + 1], nm2);
          } else {
            p01 = exp2_pair<false>(X[2 * w], nm2);
            p23 = exp2_pair<false>(X[2 * w + 1], nm2);
          }
          l2 = f2_add(l2, p01);
          l2 = f2_add(l2, p23);
          float2 q01 = f2_mul(p01, c2), q23 = f2_mul(p23, c2);
          pw[w] = e4m3x4(q01.x, q01.y, q23.x, q23.y);
        }
        tmem_st32(tS + lane_off + T::kPCol, pw);
      } else {
        uint32_t pw[2][32];
#pragma unroll
        for (int w = 0; w < 64; ++w) {
          float2 pp = ((w % 8) < kPolyPer8) ? exp2_pair<true>(X[w], nm2) : exp2_pair<false>(X[w], nm2);
          l2 = f2_add(l2, pp);
          __nv_bfloat162 pb = __floats2bfloat162_rn(pp.x, pp.y);   // .x in the low half
          pw[w >> 5][w & 31] = *reinterpret_cast<uint32_t*>(&pb);
        }
        tmem_st32(tS + lane_off + T::kPCol, pw[0]);
        tmem_st32(tS + lane_off + T::kPCol + 32, pw[1]);
      }
      const float lsum = l2.x + l2.y;
      l = l * alpha + lsum;
      m = m_new;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(barP);
    }
    // ------------------------------------------------ epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(barO, 0, abort_flag, p.status));
    if (ok) {
      tc_fence_after();
      const float fin = kFP8 ? (svmax / 448.0f) / l : 1.0f / l;
      const size_t orow = (size_t)row0 + r;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + lane_off + 32u * c, o);
        tmem_wait_ld();
        if (p.out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * 128 + 32 * c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(o[4 * e]) * fin, __uint_as_float(o[4 * e + 1]) * fin,
                                 __uint_as_float(o[4 * e + 2]) * fin,
                                 __uint_as_float(o[4 * e + 3]) * fin);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow * 128 +
                                                32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t w4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              __nv_bfloat162 pb = __floats2bfloat162_rn(__uint_as_float(o[8 * e + 2 * u]) * fin,
                                                        __uint_as_float(o[8 * e + 2 * u + 1]) * fin);
              w4[u] = *reinterpret_cast<uint32_t*>(&pb);
            }
            dst[e] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace fqa
