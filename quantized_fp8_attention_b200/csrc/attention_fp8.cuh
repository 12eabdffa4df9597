// attention_fp8.cuh -- persistent FP8 attention forward on tcgen05, with P
// staged through shared memory so that a Q tile's next S = Q K^T overlaps
// its current softmax, and each score row split between two threads.
//
// Arithmetic: the per-row rule of attention.cuh (FP8 scaled dot-product
// attention with Q, K, V as E4M3 codes and per-64-token block scales, "NVIDIA
// RTX AI optimiert FLUX.1 fuer Bilddaten mit niedriger Genauigkeit", SDPA
// quantization paragraph).
//
// Organisation (one CTA per SM, persistent over work items):
//   work item   = (b, h, pair of 128-row Q tiles); items taken round-robin
//   warps 0-15  softmax: warpgroup 2t+hf handles Q tile t, keys [64hf, 64hf+64)
//               of every KV tile (thread = row = TMEM lane)
//   warp 16     TMA producer: Q0, Q1 per item; K tiles through a ring
//   warp 17     TMEM allocator; tcgen05.mma issuer of Q tile 0
//   warp 18     TMA producer: V tiles through a ring
//   warp 19     tcgen05.mma issuer of Q tile 1
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// Shared memory: Q0, Q1; kStages K and V tiles; P_t in two buffers per Q
// tile (128 rows x 128 keys E4M3, the K-major 128-byte-swizzled layout the
// MMA reads as its A operand); the halves' row sums at the end of an item.
//
// Per KV tile g of the CTA's work, each softmax thread (row r, half hf):
//   wait S_t(g) -> tcgen05.ld the other half's 64 scores, then its own 64
//   -> row max over all 128 keys (both halves compute the same value), x,
//   alpha -> exponentials of its 64 keys (the second 32 scores read again
//   halfway, after which barSfree lets S_t(g+1) into the same columns),
//   partial l, P codes -> st.shared into P buffer g%2 -> wait for PV_t(g-1)
//   (barPV) -> rescale its 64 columns of O_t if a row maximum moved ->
//   arrive barP.
// The two halves of a row need no exchange per tile: the maximum is
// computed redundantly, the partial sums l share every alpha and are added
// once at the end of the item.
// The MMA issuer of tile t, per KV tile g: S_t(g+1) once barSfree_t(g) (and
// K(g+1)), then PV_t(g) once barP_t(g) (and V(g)).  A K stage is released
// after both tiles' S MMAs of it, a V stage after both PVs; Q after both S
// of an item's last tile (each barrier counts one commit per issuer).  None
// of these events waits on an MMA issued after it, so the fixed order cannot
// deadlock; every wait is bounded.
// Sequences of any length: the last KV tile of a head holds N % 128 keys.
// The TMA loads (3-D: channel, row within the head, head) fill rows past N
// with zeros; the K producer then overwrites the missing K rows of that tile
// with copies of key N-1 (same scale block, so the same score: the row
// maximum is unchanged), whose V rows stay zero (no term in O).  Their p
// terms in the row sum are subtracted in the epilogue, from key N-1's score
// recomputed from its codes.  The softmax loop itself carries no masking.
// Keys left out by a key mask (the keys an error-corrected pass handles
// exactly) are either masked in TMEM before the softmax reads a tile
// (kMaskable), or, when every 64-key block keeps at least one key, patched
// by the producers (kPatch): each left-out key's K row becomes a copy of the
// first kept key of its block (same codes and block scale, so the same score:
// the row maximum is unchanged) and its V row becomes zero (no term in O).
// The copies' terms stay in the row sum the kernel reports (row_stats); the
// caller takes them out (the error-corrected merge recomputes the kept keys'
// scores from the same codes), so the softmax loop is the unmasked one.
#pragma once

#include "attention.cuh"
#include "device.cuh"

namespace fqa {

constexpr int kF8Threads = 640;
// warp indices: Q/K producer, MMA issuer of tile 0 (and TMEM owner), V
// producer, MMA issuer of tile 1
constexpr int kF8Producer = 16, kF8Mma = 17, kF8ProducerV = 18, kF8Mma1 = 19;

struct F8Traits {
  static constexpr int kTileBytes = 128 * 128;                  // E4M3, 128 rows x 128 B
  static constexpr int kStages = 3;
  static constexpr uint32_t kIdescS = make_idesc(0, 0, 128, 128, 0);
  static constexpr uint32_t kIdescPV = make_idesc(0, 0, 128, 128, 1);
  static constexpr int kOffQ = 0;                                // Q0, Q1
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffP = kOffV + kStages * kTileBytes;     // [tile][buffer]
  static constexpr int kOffL = kOffP + 4 * kTileBytes;          // [item parity][tile][half][row]
  static constexpr int kOffBar = kOffL + 2 * 2 * 2 * 128 * 4;
  // fullK, fullV, emptyK, emptyV [kStages]; barQ, barQfree; barS, barSfree,
  // barP, barPV, barDrain, barL [2 each]; barPatch, barPatchV
  static constexpr int kNumBars = 4 * kStages + 2 + 12 + 2;
  static constexpr int kSmemBytes = kOffBar + 8 * kNumBars + 16 + 1024;
};

struct F8Item {
  int b, h, qp;
};

__device__ __forceinline__ F8Item f8_item(int item, int H, int npairs) {
  F8Item w;
  w.qp = item % npairs;
  const int bh = item / npairs;
  w.h = bh % H;
  w.b = bh / H;
  return w;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Maximum of 32 raw binary32 scores (two independent fmax3 chains).
__device__ __forceinline__ float max32(const uint32_t (&u)[32]) {
  float c0 = fmax3(__uint_as_float(u[0]), __uint_as_float(u[1]), __uint_as_float(u[2]));
  float c1 = fmax3(__uint_as_float(u[16]), __uint_as_float(u[17]), __uint_as_float(u[18]));
#pragma unroll
  for (int e = 3; e < 15; e += 2) {
    c0 = fmax3(c0, __uint_as_float(u[e]), __uint_as_float(u[e + 1]));
    c1 = fmax3(c1, __uint_as_float(u[16 + e]), __uint_as_float(u[16 + e + 1]));
  }
  return fmax3(c0, __uint_as_float(u[15]), fmaxf(c1, __uint_as_float(u[31])));
}

// Absent keys of a KV tile (past the end of the sequence, or excluded by a key
// mask): their scores in this thread's TMEM lane of S become -inf before the
// softmax reads them, so they drop out of the row maximum and get p = 0 (with
// a score scale a > 0, -inf * a = -inf).  pw<q>: bit k set when key 32q + k of
// the tile is present.  Both threads of a row write the same values to the
// same cells.
__device__ __forceinline__ void mask_absent_scores(uint32_t tS, uint32_t pw0, uint32_t pw1, uint32_t pw2,
                                                   uint32_t pw3) {
#pragma unroll 1
  for (int q = 0; q < 4; ++q) {
    const uint32_t present = q == 0 ? pw0 : q == 1 ? pw1 : q == 2 ? pw2 : pw3;
    if (present == ~0u) continue;
    uint32_t v[32];
    tmem_ld32(tS + 32u * (uint32_t)q, v);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (!((present >> e) & 1u)) v[e] = 0xff800000u;
    tmem_st32(tS + 32u * (uint32_t)q, v);
  }
  tmem_wait_st();
}

// kMaskable: some KV tiles may have absent keys -- the short last tile when N
// is not a multiple of 128, and keys whose bit is set in p.kmask
// ([B,H,ceil(N/32)] words, bit k of word w = key 32w + k; null = none) --
// and each row's final maximum m and sum l go to p.row_stats (if not null).
// Aligned calls without a mask use kMaskable = false, which holds no masking
// code: the full-tile loop is the same instruction stream either way only
// without it.
// kShortTail: N is not a multiple of 128 (the patched short last tile above);
// aligned calls use kShortTail = false and carry none of that code.
// kPatch: the key mask p.kmask applied by patching K and V tiles (above);
// requires N % 128 == 0 and a kept key in every 64-key block, and writes the
// row statistics like kMaskable, with l still holding the copies' terms, and
// leaves O unnormalized (O * sv_max / 448, no division by l).
template <bool kShortTail, bool kMaskable, bool kPatch = false>
__global__ void __launch_bounds__(kF8Threads, 1)
    attn_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using T = F8Traits;
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
  uint64_t* emptyK = bars + 2 * T::kStages;   // K(g) read by both S MMAs
  uint64_t* emptyV = bars + 3 * T::kStages;   // V(g) read by both PV MMAs
  uint64_t* barQ = bars + 4 * T::kStages;
  uint64_t* barQfree = barQ + 1;
  uint64_t* barS = barQ + 2;       // [2] S_t complete
  uint64_t* barSfree = barQ + 4;   // [2] S_t read by its warpgroup
  uint64_t* barP = barQ + 6;       // [2] P_t in shared memory, O_t rescaled
  uint64_t* barPV = barQ + 8;      // [2] PV_t complete
  uint64_t* barDrain = barQ + 10;  // [2] error path: an issuer's MMAs completed
  uint64_t* barL = barQ + 12;      // [2] both halves' row sums written
  uint64_t* barPatch = barQ + 14;  // a K tile to patch landed (before its patch)
  uint64_t* barPatchV = barQ + 15; // a V tile to patch landed
  float* sL = reinterpret_cast<float*>(smem + T::kOffL);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = p.N, nkv = (N + kBlockN - 1) / kBlockN, nblk = (N + 63) / 64;
  const int valid_last = N - (nkv - 1) * kBlockN;   // keys in the last KV tile
  const int npairs = (N + 2 * kBlockM - 1) / (2 * kBlockM);
  const int nitems = p.B * p.H * npairs;
  // this CTA's items and KV tiles (tile g = local item * nkv + j)
  const int my_items = nitems > (int)blockIdx.x ? (nitems - 1 - (int)blockIdx.x) / gridDim.x + 1 : 0;
  const int ntiles = my_items * nkv;
  const float c_log2e = p.softmax_scale * 1.4426950408889634f;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::kStages; ++s) {
      mbar_init(&fullK[s], 1);
      mbar_init(&fullV[s], 1);
      mbar_init(&emptyK[s], 2);              // one commit per MMA issuer
      mbar_init(&emptyV[s], 2);
    }
    mbar_init(barQ, 1);
    mbar_init(barQfree, 2);
    mbar_init(barPatch, 1);
    mbar_init(barPatchV, 1);
    mbar_init(&barDrain[0], 1);
    mbar_init(&barDrain[1], 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&barS[t], 1);
      mbar_init(&barSfree[t], 2 * kBlockM);
      mbar_init(&barP[t], 2 * kBlockM);
      mbar_init(&barPV[t], 1);
      mbar_init(&barL[t], 2 * kBlockM);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kF8Mma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kF8Producer || warp == kF8ProducerV) {
    // ------------------------------------------------ TMA producers: Q and
    // K (warp kF8Producer), V (warp kF8ProducerV); each stage of K is
    // refilled as soon as both S MMAs read it, each stage of V once both PVs
    // did
    if (lane == 0) {
      const bool is_k = warp == kF8Producer;
      const CUtensorMap* tm = is_k ? &tmK : &tmV;
      uint64_t* full = is_k ? fullK : fullV;
      uint64_t* empty = is_k ? emptyK : emptyV;
      uint8_t* ring = is_k ? sK : sV;
      if (is_k) tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(tm);
      int g = 0, pending = 0;
      uint32_t patch_phase = 0;
      bool ok = true;
      for (int it = 0; ok && it < my_items; ++it) {
        const F8Item w = f8_item((int)blockIdx.x + it * (int)gridDim.x, p.H, npairs);
        const int head = w.b * p.H + w.h;
        if (is_k) {
          if (it > 0 && !(ok = mbar_wait(barQfree, (it - 1) & 1, abort_flag, p.status))) break;
          mbar_arrive_expect_tx(barQ, 2 * T::kTileBytes);
          tma_load_3d(sQ, &tmQ, barQ, 0, w.qp * 2 * kBlockM, head);
          tma_load_3d(sQ + T::kTileBytes, &tmQ, barQ, 0, w.qp * 2 * kBlockM + kBlockM, head);
        }
        // kPatch: the key-mask words of tile j (left-out keys), loaded a tile
        // ahead so that their latency overlaps the waits and copies
        uint32_t kwn[4] = {0u, 0u, 0u, 0u};
        if constexpr (kPatch) {
#pragma unroll
          for (int q = 0; q < 4; ++q) kwn[q] = __ldg(p.kmask + (size_t)head * (N / 32) + q);
        }
        for (int j = 0; j < nkv; ++j, ++g) {
          const int s = g % T::kStages, r = g / T::kStages;
          uint32_t kw[4] = {kwn[0], kwn[1], kwn[2], kwn[3]};
          if constexpr (kPatch) {
            if (j + 1 < nkv) {
#pragma unroll
              for (int q = 0; q < 4; ++q) kwn[q] = __ldg(p.kmask + (size_t)head * (N / 32) + 4 * (j + 1) + q);
            }
          }
          if (!(ok = mbar_wait(&empty[s], (r & 1) ^ 1, abort_flag, p.status))) break;
          uint8_t* dst = ring + s * T::kTileBytes;
          if (kPatch && (kw[0] | kw[1] | kw[2] | kw[3]) != 0u) {
            // land the tile, then patch the left-out keys' rows: K rows take
            // the codes of the first kept key of their 64-key block, V rows
            // become zero; rows are 128 B with 16-byte chunk c of row x at
            // c ^ (x % 8)
            uint64_t* pbar = is_k ? barPatch : barPatchV;
            mbar_arrive_expect_tx(pbar, T::kTileBytes);
            tma_load_3d(dst, tm, pbar, 0, j * kBlockN, head);
            if (!(ok = mbar_wait(pbar, patch_phase, abort_flag, p.status))) {
              mbar_wait_drain(pbar, patch_phase);
              break;
            }
            patch_phase ^= 1u;
            for (int hb = 0; hb < 2; ++hb) {
              uint64_t left = ((uint64_t)kw[2 * hb + 1] << 32) | kw[2 * hb];
              if (left == 0) continue;
              // (a block with every key left out is excluded by the caller;
              // the index stays inside the tile regardless)
              const int f = __ffsll((long long)~left);
              const int src = 64 * hb + (f > 0 ? f - 1 : 0);
              uint4 row[8];
              if (is_k) {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                  row[c] = *reinterpret_cast<const uint4*>(dst + src * 128 + ((c ^ (src & 7)) << 4));
              } else {
#pragma unroll
                for (int c = 0; c < 8; ++c) row[c] = make_uint4(0u, 0u, 0u, 0u);
              }
              while (left != 0) {
                const int x = 64 * hb + __ffsll((long long)left) - 1;
                left &= left - 1;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                  *reinterpret_cast<uint4*>(dst + x * 128 + ((c ^ (x & 7)) << 4)) = row[c];
              }
            }
            fence_proxy_async_smem();            // generic writes -> the MMA's reads
            mbar_arrive(&full[s]);
          } else if (kShortTail && is_k && j == nkv - 1) {
            // the short last K tile: land it, then copy key N-1 (tile row
            // valid_last - 1) over the zero-filled rows past N, and only then
            // release it to the MMA.  Rows are 128 B with 16-byte chunk c of
            // row x at c ^ (x % 8) (128-byte swizzle).
            mbar_arrive_expect_tx(barPatch, T::kTileBytes);
            tma_load_3d(dst, tm, barPatch, 0, j * kBlockN, head);
            if (!(ok = mbar_wait(barPatch, patch_phase, abort_flag, p.status))) {
              mbar_wait_drain(barPatch, patch_phase);
              break;
            }
            patch_phase ^= 1u;
            const int src = valid_last - 1;
            uint4 row[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
              row[c] = *reinterpret_cast<const uint4*>(dst + src * 128 + ((c ^ (src & 7)) << 4));
            for (int x = valid_last; x < kBlockN; ++x)
#pragma unroll
              for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(dst + x * 128 + ((c ^ (x & 7)) << 4)) = row[c];
            fence_proxy_async_smem();            // generic writes -> the MMA's reads
            mbar_arrive(&full[s]);
          } else {
            mbar_arrive_expect_tx(&full[s], T::kTileBytes);
            tma_load_3d(dst, tm, &full[s], 0, j * kBlockN, head);
            pending = g + 1;
          }
        }
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA exits
        for (int q = (pending > T::kStages ? pending - T::kStages : 0); q < pending; ++q)
          mbar_wait_drain(&full[q % T::kStages], (q / T::kStages) & 1);
      }
    }
  } else if (warp == kF8Mma || warp == kF8Mma1) {
    // ------------------------------------------------ MMA issuers, one per Q
    // tile: an issuing thread is held for about as long as the tensor core
    // takes for the MMA ahead of it, so each tile gets its own
    if (lane == 0) {
      // This thread shares its sub-partition with four softmax warps, so the
      // issue path is kept short: descriptors are built once (a stage or a
      // buffer only moves the start address, the low field, in 16-byte
      // units) and the stage, phase and item counters advance without
      // divisions.
      const int t = warp == kF8Mma ? 0 : 1;
      const uint64_t dQ = make_sdesc_sw128(smem_u32(sQ) + t * T::kTileBytes, 16, 1024);
      const uint64_t dK0 = make_sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV0 = make_sdesc_sw128(smem_u32(sV), 16384, 1024);
      const uint64_t dP0 = make_sdesc_sw128(smem_u32(sP) + 2 * t * T::kTileBytes, 16, 1024);
      constexpr uint64_t kTileStep = T::kTileBytes >> 4;
      const uint32_t tS = tmem + 128u * t, tO = tmem + 256u + 128u * t;
      bool ok = true;
      // S_t(g) = Q_t K(g)^T for the tile at stage sk (phase bit kph, column
      // block jk of item ik); commits barS_t, this issuer's share of the K
      // stage release and, after an item's last KV tile, of barQfree
      int sk = 0, jk = 0, ik = 0;
      uint32_t kph = 0;
      auto issue_s = [&]() -> bool {
        if (jk == 0 && !mbar_wait(barQ, ik & 1, abort_flag, p.status)) return false;
        if (!mbar_wait(&fullK[sk], kph, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint64_t dK = dK0 + kTileStep * (uint64_t)sk;
#pragma unroll
        for (int k = 0; k < 4; ++k)              // 32 keys' worth of K per step: +32 B
          mma_f8_ss(tS, dQ + 2 * k, dK + 2 * k, T::kIdescS, k > 0);
        tc_commit(&barS[t]);
        tc_commit(&emptyK[sk]);
        if (jk == nkv - 1) tc_commit(barQfree);
        if (++sk == T::kStages) { sk = 0; kph ^= 1u; }
        if (++jk == nkv) { jk = 0; ++ik; }
        return true;
      };
      // O_t (+)= P_t(g) V(g) for the tile at stage sv (phase vph, column
      // block jv), P buffer pb; commits barPV_t and this issuer's share of
      // the V stage release
      int sv = 0, jv = 0;
      uint32_t vph = 0, pb = 0;
      auto issue_pv = [&]() -> bool {
        if (!mbar_wait(&fullV[sv], vph, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint64_t dP = dP0 + kTileStep * (uint64_t)pb;
        const uint64_t dV = dV0 + kTileStep * (uint64_t)sv;
#pragma unroll
        for (int k = 0; k < 4; ++k)              // 32 keys per step: P +32 B, V +32 rows
          mma_f8_ss(tO, dP + 2 * k, dV + 256 * k, T::kIdescPV, jv > 0 || k > 0);
        tc_commit(&barPV[t]);
        tc_commit(&emptyV[sv]);
        if (++sv == T::kStages) { sv = 0; vph ^= 1u; }
        if (++jv == nkv) jv = 0;
        pb ^= 1u;
        return true;
      };
      // per KV tile g: S_t(g+1) once the warpgroups of tile t have read
      // S_t(g), then PV_t(g) once their P_t(g) landed
      if (ntiles > 0) ok = issue_s();
      for (int g = 0; ok && g < ntiles; ++g) {
        if (g + 1 < ntiles) {
          if (!(ok = mbar_wait(&barSfree[t], g & 1, abort_flag, p.status))) break;
          if (!(ok = issue_s())) break;
        }
        if (!(ok = mbar_wait(&barP[t], g & 1, abort_flag, p.status))) break;
        if (!(ok = issue_pv())) break;
      }
      if (!ok) {
        // let the MMAs this thread issued finish before TMEM is released
        tc_commit(&barDrain[t]);
        mbar_wait_drain(&barDrain[t], 0);
      }
    }
    __syncwarp();
  } else if (warp < 16) {
    // ------------------------------------------------ softmax warpgroups
    const int t = warp >> 3;                     // Q tile of the pair
    const int hf = (warp >> 2) & 1;              // half of the keys: [64hf, 64hf+64)
    const int r = threadIdx.x & 127;             // row in tile == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + 128u * t + lane_off, tO = tmem + 256u + 128u * t + lane_off;
    // this thread's half row of the two P buffers; 16-byte chunk c of the
    // row sits at c ^ (r % 8)
    const uint32_t prow = smem_u32(sP) + (uint32_t)(2 * t) * T::kTileBytes + (uint32_t)r * 128u;
    const uint32_t sw = (uint32_t)(r & 7);
    const int nmw = (N + 31) / 32;               // key-mask words per head
    int g = 0;                                   // KV tile counter (global over items)
    bool ok = true;
    for (int it = 0; ok && it < my_items; ++it) {
      const F8Item w = f8_item((int)blockIdx.x + it * (int)gridDim.x, p.H, npairs);
      const size_t head = (size_t)w.b * p.H + w.h;
      const int qrow = w.qp * 2 * kBlockM + t * kBlockM + r;     // row within the head
      const float* skp = p.sk + head * nblk;
      const float* svp = p.sv + head * nblk;
      const float svmax = p.sv_max[head];
      const float a_row = p.sq[head * nblk + min(qrow, N - 1) / 64];
      // block scales of a tile; blocks past the end of a short sequence are
      // read clamped (their keys are absent)
      auto blk = [nblk](int J) { return (kShortTail && J >= nblk) ? nblk - 1 : J; };
      float sk0 = __ldg(skp), sk1 = __ldg(skp + blk(1)), svh = __ldg(svp + blk(hf));
      float m = -INFINITY, l = 0.0f;

      for (int j = 0; j < nkv; ++j, ++g) {
        // block constants of this tile; the next tile's are loaded ahead
        float a0 = a_row * (sk0 * c_log2e), a1 = a_row * (sk1 * c_log2e);
        float ah = hf ? a1 : a0;
        const float cpv = svmax > 0.0f ? 448.0f * (svh / svmax) : 0.0f;
        if (j + 1 < nkv) {
          sk0 = __ldg(skp + 2 * j + 2);
          sk1 = __ldg(skp + blk(2 * j + 3));
          svh = __ldg(svp + blk(2 * j + 2 + hf));
        }
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&barS[t], g & 1, abort_flag, p.status)))) break;
        tc_fence_after();
        if constexpr (kMaskable) {
          // presence of the tile's keys, 32 per word: keys the caller's mask
          // excludes (a short last tile is patched by the K producer)
          uint32_t pw0 = ~0u, pw1 = ~0u, pw2 = ~0u, pw3 = ~0u;
          if (p.kmask != nullptr) {
            const uint32_t* km = p.kmask + head * nmw + 4 * j;
            const int nw = nmw - 4 * j;
            pw0 &= ~__ldg(km);
            if (nw > 1) pw1 &= ~__ldg(km + 1);
            if (nw > 2) pw2 &= ~__ldg(km + 2);
            if (nw > 3) pw3 &= ~__ldg(km + 3);
          }
          if ((pw0 & pw1 & pw2 & pw3) != ~0u) {
            mask_absent_scores(tS, pw0, pw1, pw2, pw3);
            // -inf * 0 would be NaN: a zero scale becomes the smallest
            // positive one, which gives the present keys the same p
            // (x = S * 2^-149 is absorbed by x - m, or is 0 when S is)
            a0 = fmaxf(a0, 1.401298464e-45f);
            a1 = fmaxf(a1, 1.401298464e-45f);
            ah = hf ? a1 : a0;
          }
        }
        // raw maxima of the other half (its scores are not kept) and of this
        // half; the first 32 of this half's scores stay in registers, the
        // other 32 are read again when the exponential loop gets to them.
        // One 32-column load in flight besides sr keeps the registers low.
        uint32_t sr[32];
        float mo, mh;
        {
          const uint32_t oc = 64u * (uint32_t)(hf ^ 1), mc = 64u * (uint32_t)hf;
          uint32_t v[32];
          tmem_ld32(tS + oc, v);
          tmem_ld32(tS + mc, sr);
          tmem_wait_ld();
          mo = max32(v);
          tmem_ld32(tS + oc + 32u, v);
          tmem_wait_ld();
          mo = fmaxf(mo, max32(v));
          tmem_ld32(tS + mc + 32u, v);
          tmem_wait_ld();
          mh = fmaxf(max32(sr), max32(v));
        }
        // raw maxima of keys [0,64) and [64,128); the scales are >= 0 and
        // rounding is monotone, so the tile max of x = S * a (rounded toward
        // zero) is the rounded product of the raw max
        const float h0 = hf ? mo : mh, h1 = hf ? mh : mo;
        const float m_new = fmaxf(m, fmaxf(__fmul_rz(h0, a0), __fmul_rz(h1, a1)));
        // a tile with no key present, after tiles with none, leaves
        // m = m_new = -inf with nothing to rescale (key masks only)
        const float alpha = (kMaskable && m_new == -INFINITY) ? 1.0f : ex2_approx(m - m_new);
        // (and -inf - -inf would be NaN: with no key present, subtract 0)
        const float nm = (kMaskable && m_new == -INFINITY) ? 0.0f : -m_new;
        const float2 nm2 = make_float2(nm, nm);
        const float2 a2 = make_float2(ah, ah);
        float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const uint32_t pbuf = prow + (uint32_t)(g & 1) * T::kTileBytes;
        const float2 c2 = make_float2(cpv, cpv);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {               // 32 keys per chunk
          if (ch == 1) {
            tmem_ld32(tS + 64u * (uint32_t)hf + 32u, sr);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&barSfree[t]);           // S_t(g+1) may overwrite these columns
          }
          uint32_t pw[8];
#pragma unroll
          for (int w4 = 0; w4 < 8; ++w4) {
            // x = S * a rounded once, toward zero: a rounding ptxas cannot
            // fuse into the next step, fma(x, 1, -m), so the row maximum gets
            // p = 1 exactly and x - m is exact near the maximum
            const uint32_t* u = &sr[4 * w4];
            const float2 x01 = f2_mul_rz(make_float2(__uint_as_float(u[0]), __uint_as_float(u[1])), a2);
            const float2 x23 = f2_mul_rz(make_float2(__uint_as_float(u[2]), __uint_as_float(u[3])), a2);
            const float2 p01 = exp2_pair(x01, nm2);
            const float2 p23 = exp2_pair(x23, nm2);
            ls[0] = f2_add(ls[0], p01);
            ls[1] = f2_add(ls[1], p23);
            const float2 q01 = f2_mul(p01, c2), q23 = f2_mul(p23, c2);
            pw[w4] = e4m3x4(q01.x, q01.y, q23.x, q23.y);
          }
          const uint32_t c0 = (uint32_t)(4 * hf + 2 * ch);
          st_shared_v4(pbuf + ((c0 ^ sw) << 4), pw[0], pw[1], pw[2], pw[3]);
          st_shared_v4(pbuf + (((c0 + 1) ^ sw) << 4), pw[4], pw[5], pw[6], pw[7]);
        }
        const float2 l2 = f2_add(ls[0], ls[1]);
        if (j > 0) {
          // O_t holds PV_t(g-1) once it completed; rescale this half's
          // columns if a row maximum moved
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&barPV[t], (g - 1) & 1, abort_flag, p.status)))) break;
          tc_fence_after();
          if (__any_sync(0xffffffffu, m_new != m)) {
            const float2 al2 = make_float2(alpha, alpha);
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
              uint32_t o[32];
              const uint32_t col = 64u * (uint32_t)hf + 32u * (uint32_t)c;
              tmem_ld32(tO + col, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                float2 v = f2_mul(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), al2);
                o[e] = __float_as_uint(v.x);
                o[e + 1] = __float_as_uint(v.y);
              }
              tmem_st32(tO + col, o);
            }
            tmem_wait_st();
          }
        }
        l = l * alpha + (l2.x + l2.y);
        m = m_new;
        fence_proxy_async_smem();                // P stores -> the MMA's operand reads
        tc_fence_before();
        mbar_arrive(&barP[t]);
      }
      if (!ok) break;
      // ------------------------------------------------ epilogue: this half's columns
      float* lx = sL + ((it & 1) * 2 + t) * 2 * 128;
      lx[hf * 128 + r] = l;
      mbar_arrive(&barL[t]);
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&barL[t], it & 1, abort_flag, p.status)))) break;
      float l_row = lx[r] + lx[128 + r];
      if (kShortTail && qrow < N) {
        // the copies of key N-1 in the short last tile added 128 - valid_last
        // terms p(N-1) = 2^(x - m) to l: recompute key N-1's score from the
        // codes (E4M3 products are exact in binary32) and take them out
        const uint32_t* qa = reinterpret_cast<const uint32_t*>(p.q8 + (head * N + qrow) * 128);
        const uint32_t* ka = reinterpret_cast<const uint32_t*>(p.k8 + (head * N + N - 1) * 128);
        float sdot = 0.0f;
#pragma unroll 4
        for (int c4 = 0; c4 < 32; ++c4) {
          const uint32_t qw = __ldg(qa + c4), kw = __ldg(ka + c4);
          const float2 q01 = e4m3x2_to_f2(qw & 0xFFFFu), q23 = e4m3x2_to_f2(qw >> 16);
          const float2 k01 = e4m3x2_to_f2(kw & 0xFFFFu), k23 = e4m3x2_to_f2(kw >> 16);
          sdot = __fmaf_rn(q01.x, k01.x, sdot);
          sdot = __fmaf_rn(q01.y, k01.y, sdot);
          sdot = __fmaf_rn(q23.x, k23.x, sdot);
          sdot = __fmaf_rn(q23.y, k23.y, sdot);
        }
        const float a_last = a_row * (__ldg(skp + nblk - 1) * c_log2e);
        const float p_dup = ex2_approx(__fmaf_rn(__fmul_rz(sdot, a_last), 1.0f, -m));
        l_row -= (float)(kBlockN - valid_last) * p_dup;
      }
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&barPV[t], (g - 1) & 1, abort_flag, p.status)))) break;
      tc_fence_after();
      const bool store = qrow < N;
      // l_row = 0 only when a key mask excluded every key of the row
      // (kPatch: O leaves unnormalized, since l still holds the copies' terms)
      const float fin = kPatch ? svmax / 448.0f
                               : ((kMaskable && !(l_row > 0.0f)) ? 0.0f : (svmax / 448.0f) / l_row);
      const size_t orow = head * N + (size_t)qrow;
      if constexpr (kMaskable || kPatch) {
        if (p.row_stats != nullptr && hf == 0 && store) p.row_stats[orow] = make_float2(m, l_row);
      }
      // the output row: [B,H,N,128], or with out_P > 1 the sequence all-to-all
      // layout [B, out_P, H, N / out_P, 128] (chunk c: tokens [c N/out_P, ...))
      size_t orow_out = orow;
      if (p.out_P > 1) {
        const int nl = N / p.out_P, cq = qrow / nl;
        orow_out = (((size_t)w.b * p.out_P + cq) * p.H + w.h) * nl + (qrow - cq * nl);
      }
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        const int col = 64 * hf + 32 * c;
        tmem_ld32(tO + (uint32_t)col, o);
        tmem_wait_ld();
        if (!store) continue;
        if (p.out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow_out * 128 + col);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(o[4 * e]) * fin, __uint_as_float(o[4 * e + 1]) * fin,
                                 __uint_as_float(o[4 * e + 2]) * fin,
                                 __uint_as_float(o[4 * e + 3]) * fin);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow_out * 128 + col);
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
      // the next item's first PV overwrites O_t only after this warpgroup's
      // next barP arrival, which comes after these loads
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kF8Mma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fqa
