// attention_nvfp4.cuh -- attention with Q.K^T in NVFP4 on the block-scaled
// tensor cores and P.V in FP8 ("NVIDIA RTX AI optimiert FLUX.1 fuer
// Bilddaten mit niedriger Genauigkeit", SDPA quantization paragraph: the FP8
// and FP4 schemes differ only in the precision of the Q, K, V projections and
// attention itself stays in FP8).
//
// Arithmetic (per query row i, KV tiles of 128 keys, ascending):
//   S_ij = sum over 16-channel groups g of sfq_ig sfk_jg sum_c e2m1(q_ic) e2m1(k_jc)
//          (tcgen05.mma kind::mxf4nvf4, UE4M3 scale per 16 elements, FP32)
//   x_ij = S_ij * s1q_I * s1k_J * scale * log2(e)
// and from there the FP8 path's rule: exact running maximum per tile,
// p = 2^(x - m), P = E4M3(p * 448 * sv_J / sv_max), O += P.V (FP8), out =
// O * (sv_max / 448) / l.
//
// Organisation: the FP8 kernel's two Q tiles per CTA fill all 512 TMEM
// columns, leaving none for the scale factors, so this kernel runs one
// 128-row Q tile per work item (persistent, one CTA per SM):
//   warps 0-7  softmax: warp w handles TMEM lanes 32 (w % 4) .. and keys
//              [64 hf, 64 hf + 64) of every tile, hf = w / 4 (two threads
//              per row); each thread takes the row maximum from the raw
//              maxima of both halves (read from TMEM), so the halves exchange
//              only their row sums, once per item; warps 0-3 also write the
//              scale factors into TMEM (tcgen05.st) ahead of the MMAs that
//              read them
//   warp 8     TMA producer: Q (E2M1, 64 B rows, 64-byte swizzle) per item;
//              K (E2M1) and V (E4M3) tiles through three-stage rings
//   warp 9     TMEM owner and single-thread MMA issuer
// TMEM: S [0,128), O [128,256), SFA [256,264), SFB stage s [264+8s, 272+8s).
// Scale-factor layout (per MMA of K = 64, 4 groups): the factor of row m and
// group j sits in column base + m / 32, byte j, of lane m % 32, replicated in
// all four lane quarters; the two MMAs of K = 128 use columns base and
// base + 4.
#pragma once

#include "attention.cuh"
#include "device.cuh"

namespace fqa {

constexpr int kNvThreads = 320;
constexpr int kNvProducer = 8, kNvMma = 9;

struct NvTraits {
  static constexpr int kQKBytes = 128 * 64;                      // E2M1 tile, 128 rows x 64 B
  static constexpr int kVBytes = 128 * 128;                      // E4M3 tile
  static constexpr int kStages = 3;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQKBytes;
  static constexpr int kOffV = kOffK + kStages * kQKBytes;
  static constexpr int kOffP = kOffV + kStages * kVBytes;        // two buffers
  static constexpr int kOffL = kOffP + 2 * kVBytes;               // [item parity][half][row] row sums
  static constexpr int kOffBar = kOffL + 2 * 2 * 128 * 4;
  // fullK, fullV, emptyK, emptyV, barSFB [kStages]; barQ, barQfree, barSFA,
  // barS, barSfree, barP, barPV, barDrain, barL
  static constexpr int kNumBars = 5 * kStages + 9;
  // more than half of the SM's 228 KB: one CTA per SM, so the 512-column TMEM
  // allocation never waits for a co-resident CTA
  static constexpr int kSmemUsed = kOffBar + 8 * kNumBars + 16 + 1024;
  static constexpr int kSmemBytes = kSmemUsed < 118 * 1024 ? 118 * 1024 : kSmemUsed;
  // block-scaled instruction descriptor: A, B E2M1 (1), K-major, N = 128,
  // UE4M3 scales (0), M = 128, K = 64
  static constexpr uint32_t kIdescS = (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
  static constexpr uint32_t kIdescPV = make_idesc(0, 0, 128, 128, 1);
  static constexpr uint32_t kColS = 0, kColO = 128, kColSFA = 256, kColSFB = 264;
};

// D[tmem] (+)= A * B with per-16-element UE4M3 scale factors from TMEM
// (kind::mxf4nvf4, E2M1 operands from shared memory).
__device__ __forceinline__ void mma_nvfp4_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Shared-memory descriptor, 64-byte swizzle (layout type 4), K-major: rows of
// 64 B, 8-row groups 512 B apart.
__device__ __forceinline__ uint64_t make_sdesc_sw64(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;               // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(512u >> 4) << 32;      // stride byte offset
  d |= (uint64_t)1u << 46;               // version
  d |= (uint64_t)4u << 61;               // SWIZZLE_64B
  return d;
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

struct NvParams {
  int B, H, N;
  float softmax_scale;
  const uint8_t* sfq;    // [B,H,N,8] UE4M3 group scales of Q
  const uint8_t* sfk;    // [B,H,N,8] of smoothed K
  const float* sq1;      // [B,H,N/64] block scales
  const float* sk1;
  const float* sv;       // V: as the FP8 path
  const float* sv_max;
  void* out;
  int out_f32;
  uint32_t* status;
};

// This thread's lane of the scale factors of 128 rows starting at `row0`
// (sf: [rows][8] bytes): column (4 kk + m / 32) gets the four factors of MMA
// kk of row 32 (m / 32) + lane, so the four lane quarters hold identical
// copies.  Rows at or past `rend` (beyond the end of the sequence) get zero
// factors and are not read.
__device__ __forceinline__ void write_scale_factors(uint32_t taddr, const uint8_t* sf, size_t row0, size_t rend,
                                                    int lane) {
  uint32_t v[8];
#pragma unroll
  for (int mh = 0; mh < 4; ++mh) {
    const size_t row = row0 + 32 * mh + lane;
    const uint2 f = row < rend ? __ldg(reinterpret_cast<const uint2*>(sf + row * 8)) : make_uint2(0u, 0u);
    v[mh] = f.x;
    v[4 + mh] = f.y;
  }
  tmem_st8(taddr, v);
}

// kShortTail: N is not a multiple of 128 -- the last Q tile and the last KV
// tile are short: keys past N get x = -inf (no maximum, p or row-sum term;
// their V rows are zero-filled by the tensor map), rows past N are not
// stored.  Aligned calls use kShortTail = false and carry none of that code.
template <bool kShortTail>
__global__ void __launch_bounds__(kNvThreads, 1)
    attn_nvfp4_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const NvParams p) {
  using T = NvTraits;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + T::kOffQ;
  uint8_t* sK = smem + T::kOffK;
  uint8_t* sV = smem + T::kOffV;
  uint8_t* sP = smem + T::kOffP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::kOffBar);
  uint64_t* fullK = bars;
  uint64_t* fullV = bars + T::kStages;
  uint64_t* emptyK = bars + 2 * T::kStages;
  uint64_t* emptyV = bars + 3 * T::kStages;
  uint64_t* barSFB = bars + 4 * T::kStages;
  uint64_t* barQ = bars + 5 * T::kStages;
  uint64_t* barQfree = barQ + 1;
  uint64_t* barSFA = barQ + 2;
  uint64_t* barS = barQ + 3;
  uint64_t* barSfree = barQ + 4;
  uint64_t* barP = barQ + 5;
  uint64_t* barPV = barQ + 6;
  uint64_t* barDrain = barQ + 7;
  uint64_t* barL = barQ + 8;        // both halves' row sums of an item written
  float* sL = reinterpret_cast<float*>(smem + T::kOffL);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = p.N, nkv = (N + kBlockN - 1) / kBlockN, nblk = (N + 63) / 64;
  const int nq = (N + kBlockM - 1) / kBlockM;
  const int valid_last = N - (nkv - 1) * kBlockN;   // keys in the last KV tile
  const int nitems = p.B * p.H * nq;
  const int my_items = nitems > (int)blockIdx.x ? (nitems - 1 - (int)blockIdx.x) / gridDim.x + 1 : 0;
  const int ntiles = my_items * nkv;
  const float c_log2e = p.softmax_scale * 1.4426950408889634f;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::kStages; ++s) {
      mbar_init(&fullK[s], 1);
      mbar_init(&fullV[s], 1);
      mbar_init(&emptyK[s], 1);
      mbar_init(&emptyV[s], 1);
      mbar_init(&barSFB[s], kBlockM);
    }
    mbar_init(barQ, 1);
    mbar_init(barQfree, 1);
    mbar_init(barSFA, kBlockM);
    mbar_init(barS, 1);
    mbar_init(barSfree, 2 * kBlockM);
    mbar_init(barP, 2 * kBlockM);
    mbar_init(barL, 2 * kBlockM);
    mbar_init(barPV, 1);
    mbar_init(barDrain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kNvMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kNvProducer) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int g = 0, pending = 0;
      bool ok = true;
      for (int it = 0; ok && it < my_items; ++it) {
        const int item = (int)blockIdx.x + it * (int)gridDim.x;
        const int head = item / nq, qt = item - head * nq;
        if (it > 0 && !(ok = mbar_wait(barQfree, (it - 1) & 1, abort_flag, p.status))) break;
        mbar_arrive_expect_tx(barQ, T::kQKBytes);
        tma_load_3d(sQ, &tmQ, barQ, 0, qt * kBlockM, head);
        for (int j = 0; j < nkv; ++j, ++g) {
          const int s = g % T::kStages, r = g / T::kStages;
          if (!(ok = mbar_wait(&emptyK[s], (r & 1) ^ 1, abort_flag, p.status))) break;
          mbar_arrive_expect_tx(&fullK[s], T::kQKBytes);
          tma_load_3d(sK + s * T::kQKBytes, &tmK, &fullK[s], 0, j * kBlockN, head);
          if (!(ok = mbar_wait(&emptyV[s], (r & 1) ^ 1, abort_flag, p.status))) break;
          mbar_arrive_expect_tx(&fullV[s], T::kVBytes);
          tma_load_3d(sV + s * T::kVBytes, &tmV, &fullV[s], 0, j * kBlockN, head);
          pending = g + 1;
        }
      }
      if (*abort_flag) {
        for (int q = (pending > T::kStages ? pending - T::kStages : 0); q < pending; ++q) {
          mbar_wait_drain(&fullK[q % T::kStages], (q / T::kStages) & 1);
          mbar_wait_drain(&fullV[q % T::kStages], (q / T::kStages) & 1);
        }
      }
    }
  } else if (warp == kNvMma) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dQ = make_sdesc_sw64(smem_u32(sQ));
      const uint64_t dK0 = make_sdesc_sw64(smem_u32(sK));
      const uint64_t dV0 = make_sdesc_sw128(smem_u32(sV), 16384, 1024);
      const uint64_t dP0 = make_sdesc_sw128(smem_u32(sP), 16, 1024);
      const uint32_t tS = tmem + T::kColS, tO = tmem + T::kColO;
      bool ok = true;
      int sk = 0, jk = 0, ik = 0;
      uint32_t kph = 0;
      // S(g) = Q K(g)^T: two block-scaled MMAs of K = 64 (32 B of E2M1 each)
      auto issue_s = [&](int g) -> bool {
        if (jk == 0) {
          if (!mbar_wait(barQ, ik & 1, abort_flag, p.status)) return false;
          if (!mbar_wait(barSFA, ik & 1, abort_flag, p.status)) return false;
        }
        if (!mbar_wait(&fullK[sk], kph, abort_flag, p.status)) return false;
        if (!mbar_wait(&barSFB[sk], kph, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint64_t dK = dK0 + (uint64_t)((T::kQKBytes >> 4) * sk);
        const uint32_t sfa = tmem + T::kColSFA, sfb = tmem + T::kColSFB + 8u * (uint32_t)sk;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_nvfp4_ss(tS, dQ + 2 * kk, dK + 2 * kk, T::kIdescS, sfa + 4u * kk, sfb + 4u * kk, kk > 0);
        tc_commit(barS);
        tc_commit(&emptyK[sk]);
        if (jk == nkv - 1) tc_commit(barQfree);
        if (++sk == T::kStages) { sk = 0; kph ^= 1u; }
        if (++jk == nkv) { jk = 0; ++ik; }
        (void)g;
        return true;
      };
      int sv = 0, jv = 0;
      uint32_t vph = 0, pb = 0;
      auto issue_pv = [&]() -> bool {
        if (!mbar_wait(&fullV[sv], vph, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint64_t dP = dP0 + (uint64_t)((T::kVBytes >> 4) * pb);
        const uint64_t dV = dV0 + (uint64_t)((T::kVBytes >> 4) * sv);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_f8_ss(tO, dP + 2 * k, dV + 256 * k, T::kIdescPV, jv > 0 || k > 0);
        tc_commit(barPV);
        tc_commit(&emptyV[sv]);
        if (++sv == T::kStages) { sv = 0; vph ^= 1u; }
        if (++jv == nkv) jv = 0;
        pb ^= 1u;
        return true;
      };
      if (ntiles > 0) ok = issue_s(0);
      for (int g = 0; ok && g < ntiles; ++g) {
        if (g + 1 < ntiles) {
          if (!(ok = mbar_wait(barSfree, g & 1, abort_flag, p.status))) break;
          if (!(ok = issue_s(g + 1))) break;
        }
        if (!(ok = mbar_wait(barP, g & 1, abort_flag, p.status))) break;
        if (!(ok = issue_pv())) break;
      }
      if (!ok) {
        tc_commit(barDrain);
        mbar_wait_drain(barDrain, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax (warps 0-7)
    const int hf = warp >> 2;                    // keys [64 hf, 64 hf + 64) of each tile
    const int r = threadIdx.x & 127;             // row of the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + T::kColS + lane_off, tO = tmem + T::kColO + lane_off;
    const uint32_t prow = smem_u32(sP) + (uint32_t)r * 128u;
    const uint32_t sw = (uint32_t)(r & 7);
    const bool sf_writer = hf == 0;              // warps 0-3 write the scale factors
    // scale factors ride one step ahead of the MMAs that read them: the Q
    // factors of item it+1 go in once the last S MMA of item it completed
    // (before that S is released, so the MMA issuer never waits on a softmax
    // epilogue), the K factors of tile g+1 at the start of tile g (their
    // stage was last read by tile g-2's MMA, which has completed)
    auto item_head = [&](int i) { return ((int)blockIdx.x + i * (int)gridDim.x) / nq; };
    auto item_qt = [&](int i) { return ((int)blockIdx.x + i * (int)gridDim.x) % nq; };
    if (sf_writer && my_items > 0) {
      const size_t h0 = (size_t)item_head(0) * N;
      write_scale_factors(tmem + T::kColSFA + lane_off, p.sfq, h0 + (size_t)item_qt(0) * kBlockM, h0 + N, lane);
      write_scale_factors(tmem + T::kColSFB + lane_off, p.sfk, h0, h0 + N, lane);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(barSFA);
      mbar_arrive(&barSFB[0]);
    }
    int g = 0;
    bool ok = true;
    for (int it = 0; ok && it < my_items; ++it) {
      const int head = item_head(it), qt = item_qt(it);
      const size_t hrow = (size_t)head * N;
      const int qrow = qt * kBlockM + r;
      const float* skp = p.sk1 + (size_t)head * nblk;
      const float* svp = p.sv + (size_t)head * nblk;
      const float svmax = p.sv_max[head];
      const float a_row = p.sq1[(size_t)head * nblk + min(qrow, N - 1) / 64];
      // block scales of a tile; blocks past the end of a short sequence are
      // read clamped (their keys are absent)
      auto blk = [nblk](int J) { return (kShortTail && J >= nblk) ? nblk - 1 : J; };
      float m = -INFINITY, l = 0.0f;
      for (int j = 0; j < nkv; ++j, ++g) {
        if (sf_writer && g + 1 < ntiles) {
          // the next K tile: this item's tile j+1, or the next item's tile 0
          const size_t nh = j + 1 < nkv ? hrow : (size_t)item_head(it + 1) * N;
          const size_t nrow = j + 1 < nkv ? hrow + (size_t)(j + 1) * kBlockN : nh;
          write_scale_factors(tmem + T::kColSFB + 8u * (uint32_t)((g + 1) % T::kStages) + lane_off, p.sfk,
                              nrow, nh + N, lane);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&barSFB[(g + 1) % T::kStages]);
        }
        const float a0 = a_row * (__ldg(skp + 2 * j) * c_log2e);
        const float a1 = a_row * (__ldg(skp + blk(2 * j + 1)) * c_log2e);
        const float ah = hf ? a1 : a0;
        const float svh = __ldg(svp + blk(2 * j + hf));
        // keys of this half present in the tile (all but in a short last tile)
        const int nvh = (kShortTail && j == nkv - 1) ? min(64, max(0, valid_last - 64 * hf)) : 64;
        const int nvo = (kShortTail && j == nkv - 1) ? min(64, max(0, valid_last - 64 * (hf ^ 1))) : 64;
        const float cpv = svmax > 0.0f ? 448.0f * (svh / svmax) : 0.0f;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(barS, g & 1, abort_flag, p.status)))) break;
        tc_fence_after();
        if (sf_writer && j == nkv - 1 && it + 1 < my_items) {
          // this item's last S MMA completed: the next item's Q factors
          const size_t nh = (size_t)item_head(it + 1) * N;
          write_scale_factors(tmem + T::kColSFA + lane_off, p.sfq, nh + (size_t)item_qt(it + 1) * kBlockM, nh + N,
                              lane);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(barSFA);
        }
        // this half's 64 scores stay in registers; the other half's only give
        // their raw maximum (a >= 0 and rounding is monotone, so the maximum
        // of the rounded products is the rounded product of the raw maximum)
        uint32_t u[64];
        float mo;
        {
          uint32_t v[32];
          tmem_ld32(tS + 64u * (uint32_t)hf, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          tmem_ld32(tS + 64u * (uint32_t)hf + 32u, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tmem_ld32(tS + 64u * (uint32_t)(hf ^ 1), v);
          tmem_wait_ld();
          mo = -INFINITY;
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (!kShortTail || e < nvo) mo = fmaxf(mo, __uint_as_float(v[e]));
          tmem_ld32(tS + 64u * (uint32_t)(hf ^ 1) + 32u, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (!kShortTail || 32 + e < nvo) mo = fmaxf(mo, __uint_as_float(v[e]));
        }
        tc_fence_before();
        mbar_arrive(barSfree);                   // S may be overwritten by the next tile's MMA
        float mh = -INFINITY;
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (!kShortTail || e < nvh) mh = fmaxf(mh, __uint_as_float(u[e]));
        const float h0 = hf ? mo : mh, h1 = hf ? mh : mo;
        // (a half with no key present has raw maximum -inf: it takes no part)
        const float x0 = (kShortTail && h0 == -INFINITY) ? -INFINITY : __fmul_rz(h0, a0);
        const float x1 = (kShortTail && h1 == -INFINITY) ? -INFINITY : __fmul_rz(h1, a1);
        const float m_new = fmaxf(m, fmaxf(x0, x1));
        const float alpha = ex2_approx(m - m_new);
        float ls = 0.0f;
        const uint32_t pbuf = prow + (uint32_t)(g & 1) * T::kVBytes;
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16) {     // 16 keys: one 16-byte chunk of P
          uint32_t pw[4];
#pragma unroll
          for (int w4 = 0; w4 < 4; ++w4) {
            float pv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x = __fmul_rz(__uint_as_float(u[16 * c16 + 4 * w4 + e]), ah);
              pv[e] = (kShortTail && 16 * c16 + 4 * w4 + e >= nvh) ? 0.0f : ex2_approx(__fmaf_rn(x, 1.0f, -m_new));
              ls += pv[e];
            }
            pw[w4] = e4m3x4(pv[0] * cpv, pv[1] * cpv, pv[2] * cpv, pv[3] * cpv);
          }
          st_shared_v4(pbuf + ((((uint32_t)(4 * hf + c16)) ^ sw) << 4), pw[0], pw[1], pw[2], pw[3]);
        }
        if (j > 0) {
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(barPV, (g - 1) & 1, abort_flag, p.status)))) break;
          tc_fence_after();
          if (__any_sync(0xffffffffu, m_new != m)) {
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
              uint32_t o[32];
              const uint32_t col = 64u * (uint32_t)hf + 32u * (uint32_t)c;
              tmem_ld32(tO + col, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tO + col, o);
            }
            tmem_wait_st();
          }
        }
        l = l * alpha + ls;
        m = m_new;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(barP);
      }
      if (!ok) break;
      // ------------------------------------------------ epilogue: this half's 64 columns
      float* lx = sL + (it & 1) * 2 * 128;
      lx[hf * 128 + r] = l;
      mbar_arrive(barL);
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(barL, it & 1, abort_flag, p.status)))) break;
      const float l_row = lx[r] + lx[128 + r];
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(barPV, (g - 1) & 1, abort_flag, p.status)))) break;
      tc_fence_after();
      const float fin = (svmax / 448.0f) / l_row;
      const size_t orow = hrow + (size_t)qrow;
      const bool store = !kShortTail || qrow < N;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        const int col = 64 * hf + 32 * c;
        tmem_ld32(tO + (uint32_t)col, o);
        tmem_wait_ld();
        if (!store) continue;
        if (p.out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * 128 + col);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(o[4 * e]) * fin, __uint_as_float(o[4 * e + 1]) * fin,
                                 __uint_as_float(o[4 * e + 2]) * fin, __uint_as_float(o[4 * e + 3]) * fin);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow * 128 + col);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t w4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(o[8 * e + 2 * q]) * fin,
                                                              __uint_as_float(o[8 * e + 2 * q + 1]) * fin);
              w4[q] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            dst[e] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
      // the next item's first PV overwrites O only after this warp's next
      // barP arrival, which comes after these loads
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kNvMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fqa
