// attention_ws.cuh -- persistent, two-Q-tile BF16 attention forward on
// tcgen05: the unquantized comparison path ("FLUX 3 Image Klein Base",
// section "왜 이런 차이가 나나": VANILLA BF16 attention on B200), with the
// per-row online softmax of attention.cuh minus the scales and the P
// quantization (P in BF16, out = O / l).
//
// Organisation (one CTA per SM, persistent over work items):
//   work item   = (b, h, pair of 128-row Q tiles); items taken round-robin
//   warps 0-3   softmax warpgroup of Q tile 0 (thread = row = TMEM lane)
//   warps 4-7   softmax warpgroup of Q tile 1
//   warp 8      TMA producer: Q0, Q1 per item; K and V tiles through a ring
//   warp 9      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 10-11 idle
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512);
// P_t (BF16, 64 columns) overwrites the top of S_t once softmax t holds S_t
// in registers.  A BF16 tile row is 256 B: every tile is two 64-column
// halves of 128-byte-swizzled rows.
// MMA issue order per KV tile j:  PV0(j), S0(j+1), PV1(j), S1(j+1)  -- the
// tensor cores work on one tile while the other tile's softmax runs, and each
// S_t(j+1) is issued after the PV_t(j) that reads P_t(j) from the same TMEM
// columns (tcgen05.mma operations of one thread execute in issue order).  The
// commit that signals S_t(j+1) also covers PV_t(j), so once softmax t sees
// S_t(j+1) it may rescale O_t.  The two softmax warpgroups take turns for
// their exponential loops.
// Sequences of any length: TMA loads are 3-D (channel, row within the head,
// head), rows past N read as zeros, and the last KV tile's keys past N get
// raw score -inf, so p = 0 for them (the scale here is always > 0).
#pragma once

#include "attention.cuh"
#include "device.cuh"

namespace fqa {

constexpr int kWsThreads = 384;
constexpr int kPairRows = 2 * kBlockM;

struct BfTraits {
  static constexpr int kTileBytes = kBlockM * kHeadDim * 2;       // BF16
  static constexpr int kStages = 2;
  static constexpr int kKStep = 16;                                // keys per MMA K step
  static constexpr int kSteps = 128 / kKStep;
  static constexpr uint32_t kFmt = 1u;                             // BF16 operands
  static constexpr uint32_t kPCol = 64u;                           // P_t in S_t columns [64,128)
  static constexpr uint32_t kIdescS = make_idesc(kFmt, kFmt, 128, 128, 0);
  static constexpr uint32_t kIdescPV = make_idesc(kFmt, kFmt, 128, 128, 1);
  static constexpr int kOffQ = 0;                                  // Q0, Q1
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  // fullK, fullV, empty [kStages]; barQ, barQfree, barS[2], barP[2], barO[2],
  // barTurn[2]
  static constexpr int kNumBars = 3 * kStages + 10;
  static constexpr int kSmemBytes = kOffBar + 8 * kNumBars + 16 + 1024;
};

struct WsItem {
  int b, h, qp;
};

__device__ __forceinline__ WsItem ws_item(int item, int H, int npairs) {
  WsItem w;
  w.qp = item % npairs;
  const int bh = item / npairs;
  w.h = bh % H;
  w.b = bh / H;
  return w;
}

// 32 lanes x 32 bit, 8 consecutive columns.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__global__ void __launch_bounds__(kWsThreads, 1)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using T = BfTraits;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + T::kOffQ;
  uint8_t* sK = smem + T::kOffK;
  uint8_t* sV = smem + T::kOffV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::kOffBar);
  uint64_t* fullK = bars;
  uint64_t* fullV = bars + T::kStages;
  uint64_t* empty = bars + 2 * T::kStages;
  uint64_t* barQ = bars + 3 * T::kStages;
  uint64_t* barQfree = barQ + 1;
  uint64_t* barS = barQ + 2;   // [2]
  uint64_t* barP = barQ + 4;   // [2]
  uint64_t* barO = barQ + 6;   // [2]
  uint64_t* barTurn = barQ + 8;  // [2] exponential-phase turns of the two softmax warpgroups
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = p.N, nkv = (N + kBlockN - 1) / kBlockN;
  const int valid_last = N - (nkv - 1) * kBlockN;   // keys in the last KV tile
  const int npairs = (N + kPairRows - 1) / kPairRows;
  const int nitems = p.B * p.H * npairs;
  const float c_log2e = p.softmax_scale * 1.4426950408889634f;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::kStages; ++s) {
      mbar_init(&fullK[s], 1);
      mbar_init(&fullV[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(barQ, 1);
    mbar_init(barQfree, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&barS[t], 1);
      mbar_init(&barP[t], kBlockM);
      mbar_init(&barO[t], 1);
      mbar_init(&barTurn[t], kBlockM);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int g = 0, it = 0, pending = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < nitems; item += gridDim.x, ++it) {
        const WsItem w = ws_item(item, p.H, npairs);
        const int head = w.b * p.H + w.h;
        if (it > 0 && !(ok = mbar_wait(barQfree, (it - 1) & 1, abort_flag, p.status))) break;
        mbar_arrive_expect_tx(barQ, 2 * T::kTileBytes);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int y = w.qp * kPairRows + t * kBlockM;
          uint8_t* dst = sQ + t * T::kTileBytes;
          tma_load_3d(dst, &tmQ, barQ, 0, y, head);
          tma_load_3d(dst + 16384, &tmQ, barQ, 64, y, head);
        }
        for (int j = 0; j < nkv; ++j, ++g) {
          const int s = g % T::kStages, r = g / T::kStages;
          if (!(ok = mbar_wait(&empty[s], (r & 1) ^ 1, abort_flag, p.status))) break;
          const int y = j * kBlockN;
          mbar_arrive_expect_tx(&fullK[s], T::kTileBytes);
          mbar_arrive_expect_tx(&fullV[s], T::kTileBytes);
          uint8_t* dk = sK + s * T::kTileBytes;
          uint8_t* dv = sV + s * T::kTileBytes;
          tma_load_3d(dk, &tmK, &fullK[s], 0, y, head);
          tma_load_3d(dv, &tmV, &fullV[s], 0, y, head);
          tma_load_3d(dk + 16384, &tmK, &fullK[s], 64, y, head);
          tma_load_3d(dv + 16384, &tmV, &fullV[s], 64, y, head);
          pending = g + 1;
        }
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA exits
        for (int q = (pending > T::kStages ? pending - T::kStages : 0); q < pending; ++q) {
          mbar_wait_drain(&fullK[q % T::kStages], (q / T::kStages) & 1);
          mbar_wait_drain(&fullV[q % T::kStages], (q / T::kStages) & 1);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      // descriptors are built once; a K step only moves the start address,
      // which lives in the low bits (added in 16-byte units)
      const uint64_t dQ[2] = {make_sdesc_sw128(smem_u32(sQ), 16, 1024),
                              make_sdesc_sw128(smem_u32(sQ + T::kTileBytes), 16, 1024)};
      const uint32_t tS[2] = {tmem, tmem + 128};
      const uint32_t tO[2] = {tmem + 256, tmem + 384};
      int g = 0, it = 0, np[2] = {0, 0};
      bool ok = true;
      auto kstep_kmajor = [](int k) -> uint64_t {     // K-major operand, bytes >> 4:
        return (uint64_t)((k >> 2) * 1024 + (k & 3) * 2);   // 32 B per step, 16 KB per half
      };
      auto issue_s = [&](int t, uint64_t dK) {
#pragma unroll
        for (int k = 0; k < T::kSteps; ++k) {
          const uint64_t off = kstep_kmajor(k);
          mma_bf16_ss(tS[t], dQ[t] + off, dK + off, T::kIdescS, k > 0);
        }
        tc_commit(&barS[t]);
      };
      auto issue_pv = [&](int t, uint64_t dV, bool acc) {
#pragma unroll
        for (int k = 0; k < T::kSteps; ++k) {
          const uint32_t aP = tS[t] + T::kPCol + 8u * (uint32_t)k;
          const uint64_t off = (uint64_t)(k * T::kKStep * 128 / 16);   // kKStep keys x 128 B
          mma_bf16_ts(tO[t], aP, dV + off, T::kIdescPV, (acc || k > 0));
        }
      };
      auto dK_of = [&](int s_) { return make_sdesc_sw128(smem_u32(sK + s_ * T::kTileBytes), 16, 1024); };
      auto dV_of = [&](int s_) {
        return make_sdesc_sw128(smem_u32(sV + s_ * T::kTileBytes), 16384, 1024);
      };
      for (int item = blockIdx.x; ok && item < nitems; item += gridDim.x, ++it) {
        if (!(ok = mbar_wait(barQ, it & 1, abort_flag, p.status))) break;
        {
          const int s = g % T::kStages, r = g / T::kStages;
          if (!(ok = mbar_wait(&fullK[s], r & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint64_t dK = dK_of(s);
          issue_s(0, dK);
          issue_s(1, dK);
        }
        for (int j = 0; j < nkv; ++j, ++g) {
          const int s = g % T::kStages, r = g / T::kStages;
          const int s1 = (g + 1) % T::kStages, r1 = (g + 1) / T::kStages;
          const uint64_t dV = dV_of(s), dK1 = dK_of(s1);
          const bool more = j + 1 < nkv;
          // the operand tiles usually landed long ago: wait for them before P
          if (!(ok = mbar_wait(&fullV[s], r & 1, abort_flag, p.status))) break;
          if (more && !(ok = mbar_wait(&fullK[s1], r1 & 1, abort_flag, p.status))) break;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (!(ok = mbar_wait(&barP[t], np[t] & 1, abort_flag, p.status))) break;
            ++np[t];
            tc_fence_after();
            issue_pv(t, dV, j > 0);
            if (more)
              issue_s(t, dK1);
            else
              tc_commit(&barO[t]);
          }
          if (!ok) break;
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(barQfree);
      }
      if (!ok) {
        // let the MMAs this thread issued finish before TMEM is released
        tc_commit(barQfree);
        mbar_wait_drain(barQfree, it & 1);
      }
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------ softmax warpgroups
    const int t = warp >> 2;                     // Q tile of the pair
    const int r = threadIdx.x & 127;             // row in tile == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + 128u * t, tO = tmem + 256u + 128u * t;
    int ns = 0, it = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < nitems; item += gridDim.x, ++it) {
      const WsItem w = ws_item(item, p.H, npairs);
      const size_t head = (size_t)w.b * p.H + w.h;
      const int qrow = w.qp * kPairRows + t * kBlockM + r;    // row within the head
      float m = -INFINITY, l = 0.0f;
      for (int j = 0; j < nkv; ++j, ++ns) {
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&barS[t], ns & 1, abort_flag, p.status)))) break;
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + lane_off + 32u * c, sr[c]);
        tmem_wait_ld();
        if (j == nkv - 1 && valid_last < kBlockN) {
          // keys past the end of the sequence: raw score -inf, so p = 0
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (32 * c + e >= valid_last) sr[c][e] = 0xff800000u;
        }
        const float a0 = c_log2e, a1 = c_log2e;
        // maxima of the raw scores per 64-key half (8 independent chains);
        // the scales are >= 0 and rounding is monotone, so the tile max of
        // x = S * a (rounded toward zero) is the rounded product of the max
        float cm[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t* v = &sr[q >> 1][(q & 1) * 16];
          cm[q] = fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
          for (int u = 3; u < 15; u += 2) cm[q] = fmax3(cm[q], __uint_as_float(v[u]), __uint_as_float(v[u + 1]));
          cm[q] = fmaxf(cm[q], __uint_as_float(v[15]));
        }
        const float h0 = fmaxf(fmax3(cm[0], cm[1], cm[2]), cm[3]);
        const float h1 = fmaxf(fmax3(cm[4], cm[5], cm[6]), cm[7]);
        // x = S * a rounded once, toward zero: a rounding ptxas cannot fuse
        // into the next step, fma(x, 1, -m), so the row maximum gets p = 1
        // exactly and x - m is exact near the maximum
        float2 X[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const float a = (e < 32) ? a0 : a1;
          X[e] = f2_mul_rz(make_float2(__uint_as_float(sr[e >> 4][(2 * e) & 31]),
                                       __uint_as_float(sr[e >> 4][(2 * e + 1) & 31])),
                           make_float2(a, a));
        }
        const float m_new = fmaxf(m, fmaxf(__fmul_rz(h0, a0), __fmul_rz(h1, a1)));
        const float alpha = ex2_approx(m - m_new);
        const float2 nm2 = make_float2(-m_new, -m_new);
        // Ping-pong: the two warpgroups take turns for the exponential loop
        // (MUFU-bound), so each has the sub-partitions' ex2 units to itself
        // while the tensor cores run the other tile's MMAs.  Warpgroup 0 goes
        // first; turn k of warpgroup 1 follows turn k of warpgroup 0.
        if (t == 1 || ns > 0) {
          const uint32_t par = (t == 0) ? ((ns - 1) & 1) : (ns & 1);
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&barTurn[t], par, abort_flag, p.status)))) break;
        }
        float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        {
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t pw[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const int e = 16 * ch + u;
              const float2 pp = exp2_pair(X[e], nm2);
              ls[u & 1] = f2_add(ls[u & 1], pp);
              __nv_bfloat162 pb = __floats2bfloat162_rn(pp.x, pp.y);
              pw[u] = *reinterpret_cast<uint32_t*>(&pb);
            }
            tmem_st16(tS + lane_off + T::kPCol + 16u * ch, pw);
          }
        }
        mbar_arrive(&barTurn[t ^ 1]);                // hand the turn to the other tile
        const float2 l2 = f2_add(ls[0], ls[1]);
        // O correction (O_t is stable: its last P.V completed before S_t(j))
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
        l = l * alpha + (l2.x + l2.y);
        m = m_new;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&barP[t]);
      }
      if (!ok) break;
      // ------------------------------------------------ epilogue of tile t
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&barO[t], it & 1, abort_flag, p.status)))) break;
      tc_fence_after();
      const bool store = qrow < N;
      const float fin = 1.0f / l;
      const size_t orow = head * N + (size_t)qrow;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + lane_off + 32u * c, o);
        tmem_wait_ld();
        if (!store) continue;
        if (p.out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * 128 + 32 * c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(o[4 * e]) * fin, __uint_as_float(o[4 * e + 1]) * fin,
                                 __uint_as_float(o[4 * e + 2]) * fin,
                                 __uint_as_float(o[4 * e + 3]) * fin);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow * 128 + 32 * c);
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
      // the next item's first P.V overwrites O_t only after this warpgroup's
      // next barP arrival, which comes after these loads
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fqa
