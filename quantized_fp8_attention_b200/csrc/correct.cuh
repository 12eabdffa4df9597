// correct.cuh -- error-corrected FP8 attention: FP8 attention that corrects
// only the tokens with large error ("FLUX 3 Image Klein Base: 생성 3.46배,
// 8장 확장 병목", section "왜 이런 차이가 나나": VC-Attention FP8, rho = 0.005,
// one of the B200 FP8 attention backends measured there).
//
// Readings (the page gives the name, the idea and rho only):
//  - the tokens are key/value tokens; a key's error is its own quantization
//    error e_j, the squared distance between the smoothed key and its
//    dequantized code (computed by the quantizer, pinned order);
//  - per (b, h) the kc = ceil(rho * N) keys with the largest e_j are corrected
//    (ties to the lower token index);
//  - the FP8 rule runs over the other keys (attn_fp8_kernel with a key mask,
//    FP32 output and per-row maximum m1 and sum l1); the corrected keys' part
//    is exact: s_j = (q_i . k_j - q_i . mu) * scale * log2(e) on the BF16
//    inputs (the smoothed keys, so both parts share one per-row offset),
//    m2 = max s_j, p_j = 2^(s_j - m2), l2 = sum p_j, A2 = sum p_j v_j;
//  - merge: M = max(m1, m2), w1 = 2^(m1 - M), w2 = 2^(m2 - M),
//    out = (O1 l1 w1 + A2 w2) / (l1 w1 + l2 w2).
//
// select_keys_kernel: one CTA per (b, h); radix select of the kc-th largest
// error (errors are >= 0, so their bit patterns order like their values),
// then one ordered pass writing the key mask (bit set = corrected) and the
// corrected indices in ascending order.
//
// correct_kernel: the exact part and the merge on tcgen05.  One CTA per
// (split, head) loops over the head's 128-row Q tiles; the corrected K and V
// rows (BF16) are gathered into shared memory in the layout the MMAs read
// (128-byte swizzle, two 64-channel halves), 128 keys per chunk (once per CTA
// when kc <= 128).  S = Q K_c^T (kind::f16, FP32 in TMEM); the row threads
// take S - q.mu, the exponentials and the row sum in FP32 and write P split
// into BF16 hi + lo parts (p = hi + lo to about 2^-16), so O = P_hi V + P_lo V
// keeps the exact part near FP32 precision; the epilogue merges with the FP8
// part's row and writes the output.
#pragma once

#include "attention.cuh"
#include "device.cuh"

namespace fqa {

// ------------------------------------------------------------ selection

constexpr int kSelThreads = 1024;
constexpr int kSelStageMax = 32768;   // heads up to this length are staged in shared memory (128 KB)

__global__ void __launch_bounds__(kSelThreads, 1)
    select_keys_kernel(const float* __restrict__ err, int N, int kc, uint32_t* __restrict__ kmask,
                       int* __restrict__ idx, int staged) {
  extern __shared__ uint32_t sel_stage[];
  const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const uint32_t* eg = reinterpret_cast<const uint32_t*>(err) + (size_t)bh * N;
  // the head's errors, read five times below: from shared memory when they fit
  if (staged) {
    for (int i = tid; i < N; i += kSelThreads) sel_stage[i] = __ldg(eg + i);
    __syncthreads();
  }
  const uint32_t* e = staged ? sel_stage : eg;
  const int nw = (N + 31) / 32;
  uint32_t* km = kmask + (size_t)bh * nw;
  int* id = idx + (size_t)bh * (size_t)kc;
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_want;
  __shared__ int s_cnt[2][32];
  __shared__ int s_base[2];

  // threshold T: the kc-th largest bit pattern (kc >= 1 here)
  if (tid == 0) {
    s_prefix = 0;
    s_mask = 0;
    s_want = kc;
  }
  __syncthreads();
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += kSelThreads) hist[b] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int i = tid; i < N; i += kSelThreads) {
      const uint32_t u = e[i];
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (wid == 0) {
      // the digit: walking the bins from 255 down, the first where the count
      // so far reaches `want`; lane l holds bins 255 - 8l .. 248 - 8l
      const int want = s_want;
      int c[8], tot = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        c[q] = (int)hist[255 - 8 * lane - q];
        tot += c[q];
      }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t hit = __ballot_sync(0xffffffffu, incl >= want);
      if (lane == __ffs(hit) - 1) {
        int cum = incl - tot, digit = 255 - 8 * lane;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (cum + c[q] >= want) {
            digit = 255 - 8 * lane - q;
            break;
          }
          cum += c[q];
        }
        s_want = want - cum;                    // still needed among this digit
        s_prefix = prefix | ((uint32_t)digit << shift);
        s_mask = mask | (255u << shift);
      }
    }
    __syncthreads();
  }
  const uint32_t T = s_prefix;
  const int take_eq = s_want;                   // keys equal to T to take, lowest index first

  // ordered pass: 1024 keys at a time, ranks by warp ballots and a scan
  if (tid == 0) {
    s_base[0] = 0;                              // keys equal to T seen so far
    s_base[1] = 0;                              // keys selected so far
  }
  __syncthreads();
  for (int base = 0; base < N; base += kSelThreads) {
    const int i = base + tid;
    const uint32_t u = i < N ? e[i] : 0u;
    const bool gt = i < N && u > T, eq = i < N && u == T;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const uint32_t beq = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) s_cnt[0][wid] = __popc(beq);
    __syncthreads();
    int eq_before = s_base[0];
    for (int w = 0; w < wid; ++w) eq_before += s_cnt[0][w];
    const bool sel = gt || (eq && eq_before + __popc(beq & lt_mask) < take_eq);
    const uint32_t bsel = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) {
      s_cnt[1][wid] = __popc(bsel);
      if (base + 32 * wid < N) km[(base >> 5) + wid] = bsel;
    }
    __syncthreads();
    int sel_before = s_base[1];
    for (int w = 0; w < wid; ++w) sel_before += s_cnt[1][w];
    if (sel) id[sel_before + __popc(bsel & lt_mask)] = i;
    __syncthreads();
    if (tid == 0) {
      int te = 0, ts = 0;
      for (int w = 0; w < kSelThreads / 32; ++w) {
        te += s_cnt[0][w];
        ts += s_cnt[1][w];
      }
      s_base[0] += te;
      s_base[1] += ts;
    }
    __syncthreads();
  }
}

// ------------------------------------------------- patched FP8 part's row sums

// When the FP8 part ran with patched tiles (attn_fp8_kernel<.., kPatch>: each
// corrected key's K row a copy of the first kept key of its 64-key block, its
// V row zero), its reported row sum l holds one extra term 2^(x_src - m) per
// corrected key, x_src the copied key's score.  dup_sum_kernel takes them out:
// one CTA per (128-row Q tile, head) scores the tile's rows against the copied
// keys with the same FP8 MMA on the same codes (so the same S), forms x and p
// exactly as the FP8 softmax does, and writes l - sum_J cnt_J p(src_J) back
// into the row statistics.  Needs N % 128 == 0 and fewer than 64 corrected
// keys per head (a kept key in every block; at most 63 copied keys).
constexpr int kDupThreads = 160;     // warps 0-3: one row each thread; warp 4: lists, TMA, MMA
constexpr int kDupSmem = 28 * 1024;  // Q8 16 KB + source rows 8 KB; eight CTAs per SM (8 x 64 TMEM columns)

struct DupParams {
  const uint8_t* k8;        // E4M3 codes [B,H,N,128]
  const float* sq;          // [B,H,N/64]
  const float* sk;
  const uint32_t* kmask;    // [B,H,N/32] corrected keys
  float2* stats;            // (m, l) per row [B,H,N], l corrected in place
  int N;
  float softmax_scale;
  uint32_t* status;
};

__global__ void __launch_bounds__(kDupThreads)
    dup_sum_kernel(const __grid_constant__ CUtensorMap tmQ8, const DupParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ8 = smem;                         // 128 rows x 128 B, 128-byte swizzle
  uint8_t* sKs = smem + 16384;                 // 64 rows x 128 B, 128-byte swizzle
  __shared__ uint64_t barQ, barS;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int s_src[64], s_cnt[64], s_blk[64], s_n;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tq = blockIdx.x, head = blockIdx.y, N = p.N, nblk = N / 64;
  const size_t hbase = (size_t)head * N;
  if (threadIdx.x == 0) {
    mbar_init(&barQ, 1);
    mbar_init(&barS, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 4) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&barQ, 16384);
      tma_load_3d(sQ8, &tmQ8, &barQ, 0, tq * 128, head);
    }
    __syncwarp();
    tmem_alloc(&tmem_slot, 64);
    tmem_relinquish();
    // blocks with corrected keys, ascending: the key they copy and their count
    int n = 0;
    for (int b0 = 0; b0 < nblk; b0 += 32) {
      const int J = b0 + lane;
      int cnt = 0, src = 0;
      if (J < nblk) {
        const uint32_t w0 = __ldg(p.kmask + hbase / 32 + 2 * J), w1 = __ldg(p.kmask + hbase / 32 + 2 * J + 1);
        cnt = __popc(w0) + __popc(w1);
        const int f = __ffsll((long long)~(((uint64_t)w1 << 32) | w0));
        src = 64 * J + (f > 0 ? f - 1 : 0);
      }
      const uint32_t any = __ballot_sync(0xffffffffu, cnt > 0);
      const int pos = n + __popc(any & ((1u << lane) - 1u));
      if (cnt > 0 && pos < 64) {
        s_src[pos] = src;
        s_cnt[pos] = cnt;
        s_blk[pos] = J;
      }
      n += __popc(any);
    }
    if (lane == 0) s_n = n < 64 ? n : 64;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const int nsrc = s_n;
  // the copied keys' code rows (zero rows past nsrc)
  for (int w = threadIdx.x; w < 64 * 8; w += kDupThreads) {
    const int x = w >> 3, c = w & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (x < nsrc) v = __ldg(reinterpret_cast<const uint4*>(p.k8 + (hbase + (size_t)s_src[x]) * 128) + c);
    *reinterpret_cast<uint4*>(sKs + x * 128 + ((c ^ (x & 7)) << 4)) = v;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  if (warp == 4) {
    if (lane == 0) {
      if (mbar_wait(&barQ, 0, &abort_flag, p.status)) {
        tc_fence_after();
        const uint64_t dQ = make_sdesc_sw128(smem_u32(sQ8), 16, 1024);
        const uint64_t dK = make_sdesc_sw128(smem_u32(sKs), 16, 1024);
        constexpr uint32_t kIdesc = make_idesc(0, 0, 128, 64, 0);
#pragma unroll
        for (int k = 0; k < 4; ++k) mma_f8_ss(tmem, dQ + 2 * k, dK + 2 * k, kIdesc, k > 0);
      }
      tc_commit(&barS);
    }
    __syncwarp();
  } else {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&barS, 0, &abort_flag, p.status));
    tc_fence_after();
    uint32_t u0[32], u1[32];
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    tmem_ld32(tmem + lane_off, u0);
    tmem_ld32(tmem + lane_off + 32u, u1);
    tmem_wait_ld();
    const int r = threadIdx.x;
    const size_t row = hbase + (size_t)tq * 128 + r;
    if (ok && !abort_flag) {
      const float2 st = p.stats[row];
      const float c_log2e = p.softmax_scale * 1.4426950408889634f;
      const float a_row = __ldg(p.sq + (size_t)head * nblk + (tq * 128 + r) / 64);
      const float nm = -st.x;
      float dup = 0.0f;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        if (i < nsrc) {
          // x and p as the FP8 softmax forms them: x = S * a rounded toward
          // zero, p = 2^(x - m)
          const float a = a_row * (__ldg(p.sk + (size_t)head * nblk + s_blk[i]) * c_log2e);
          const float x = __fmul_rz(__uint_as_float(i < 32 ? u0[i] : u1[i - 32]), a);
          dup = __fmaf_rn((float)s_cnt[i], ex2_approx(__fmaf_rn(x, 1.0f, nm)), dup);
        }
      }
      p.stats[row] = make_float2(st.x, st.y - dup);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// ------------------------------------------------------- exact part + merge

constexpr int kCorrThreads = 160;    // warps 0-3: one row each thread; warp 4: TMA, TMEM, MMA
constexpr int kCorrIssuer = 4;

// kKeys: corrected keys per chunk (128, or 64 when kc <= 64: half the shared
// memory, so two CTAs share an SM).
template <int kKeys>
struct CorrTraits {
  static constexpr int kQBytes = 128 * 128 * 2;                   // BF16 Q tile, two 64-channel halves
  static constexpr int kKVHalf = kKeys * 128;                     // one 64-channel half of K_c or V_c
  static constexpr int kPBytes = 128 * kKeys * 2;                 // P (hi or lo): 64-key halves of 16 KB
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + 2 * kKVHalf;
  static constexpr int kOffPhi = kOffV + 2 * kKVHalf;
  static constexpr int kOffPlo = kOffPhi + kPBytes;
  static constexpr int kOffBar = kOffPlo + kPBytes;
  static constexpr int kNumBars = 4;                               // barQ, barS, barP, barPV
  static constexpr int kSmemBytes = kOffBar + 8 * kNumBars + 16 + 1024;
  static constexpr int kCtasPerSm = kKeys == 64 ? 2 : 1;
  static constexpr uint32_t kIdescS = make_idesc(1, 1, 128, kKeys, 0);
  static constexpr uint32_t kIdescPV = make_idesc(1, 1, 128, 128, 1);
};

struct CorrParams {
  const __nv_bfloat16* q;   // BF16 inputs [B,H,N,128]
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* k_mean;      // [B,H,128]
  const int* idx;           // [B,H,kc] corrected keys, ascending
  const float* o1;          // FP8 part's FP32 output [B,H,N,128]: normalized by l1, or not (o1_raw)
  const float2* stats;      // FP8 part's (m1, l1) per row [B,H,N]
  int o1_raw;               // o1 is unnormalized (the patched FP8 part)
  void* out;                // [B,H,N,128] BF16 or FP32
  int out_f32;
  int B, H, N, kc;
  float softmax_scale;
  uint32_t* status;
};

// 16-byte chunk c (8 BF16 values) of row x of an operand tile stored as two
// 64-column halves `half` bytes apart, 128 B per row, chunk c of a half at
// c ^ (x % 8) (128-byte swizzle).
__device__ __forceinline__ uint32_t tile_chunk_off(int x, int c, int half) {
  return (uint32_t)((c >> 3) * half + x * 128 + (((c & 7) ^ (x & 7)) << 4));
}

template <int kKeys>
__global__ void __launch_bounds__(kCorrThreads, CorrTraits<kKeys>::kCtasPerSm)
    correct_kernel(const __grid_constant__ CUtensorMap tmQ, const CorrParams p) {
  using T = CorrTraits<kKeys>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + T::kOffQ;
  uint8_t* sK = smem + T::kOffK;
  uint8_t* sV = smem + T::kOffV;
  uint8_t* sPhi = smem + T::kOffPhi;
  uint8_t* sPlo = smem + T::kOffPlo;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::kOffBar);
  uint64_t* barQ = bars;
  uint64_t* barS = bars + 1;
  uint64_t* barP = bars + 2;
  uint64_t* barPV = bars + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.y, N = p.N, kc = p.kc;
  const int ntq = (N + 127) / 128, nch = (kc + kKeys - 1) / kKeys;
  // 64-key instance: q . mu from the S MMA (K_c rows 61..63 hold mu), so
  // kc <= 61 there; the 128-key one sums q . mu per row thread
  constexpr bool kMuRows = kKeys == 64;
  const float c_log2e = p.softmax_scale * 1.4426950408889634f;
  const size_t hbase = (size_t)head * N;

  if (threadIdx.x == 0) {
    mbar_init(barQ, 1);
    mbar_init(barS, 1);
    mbar_init(barP, 128);
    mbar_init(barPV, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kCorrIssuer) {
    tmem_alloc(tmem_slot, 256);               // S [0,kKeys), O [128,256)
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // corrected keys [kKeys ch, kKeys ch + kKeys) of this head -> sK, sV (zero
  // rows past kc), all threads; made visible to the tensor core
  auto gather = [&](int ch) {
    const int* ids = p.idx + (size_t)head * kc + kKeys * ch;
    const int nk = min(kKeys, kc - kKeys * ch);
    for (int w = threadIdx.x; w < kKeys * 16; w += kCorrThreads) {
      const int x = w >> 4, c = w & 15;
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (x < nk) {
        const size_t row = hbase + (size_t)__ldg(ids + x);
        kv = __ldg(reinterpret_cast<const uint4*>(p.k + row * 128) + c);
        vv = __ldg(reinterpret_cast<const uint4*>(p.v + row * 128) + c);
      } else if (kMuRows && x >= kKeys - 3) {
        // mu = hi + mid + lo in BF16 (mu - hi - mid - lo is below 2^-24 |mu|),
        // so that the S MMA also gives q . mu in its last three columns
        const int part = x - (kKeys - 3);
        const float* mu = p.k_mean + (size_t)head * 128 + 8 * c;
        uint32_t wv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float pr[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float m0 = __ldg(mu + 2 * e + h);
            const float hi = __bfloat162float(__float2bfloat16_rn(m0));
            const float mid = __bfloat162float(__float2bfloat16_rn(m0 - hi));
            const float lo = __bfloat162float(__float2bfloat16_rn((m0 - hi) - mid));
            pr[h] = part == 0 ? hi : (part == 1 ? mid : lo);
          }
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(pr[0], pr[1]);
          wv[e] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        kv = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      }
      *reinterpret_cast<uint4*>(sK + tile_chunk_off(x, c, T::kKVHalf)) = kv;
      *reinterpret_cast<uint4*>(sV + tile_chunk_off(x, c, T::kKVHalf)) = vv;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
  };
  if (nch == 1) gather(0);

  // the first Q tile; later ones are loaded as soon as the last S MMA of the
  // tile before has read sQ
  if (warp == kCorrIssuer && lane == 0 && (int)blockIdx.x < ntq) {
    mbar_arrive_expect_tx(barQ, T::kQBytes);
    tma_load_3d(sQ, &tmQ, barQ, 0, (int)blockIdx.x * 128, head);
    tma_load_3d(sQ + 16384, &tmQ, barQ, 64, (int)blockIdx.x * 128, head);
  }
  uint32_t ph_q = 0, ph_s = 0, ph_p = 0, ph_pv = 0;
  bool ok = true;
  for (int tq = blockIdx.x; tq < ntq; tq += gridDim.x) {
    const int r = threadIdx.x & 127;           // row of the tile (row threads)
    const int qrow = tq * 128 + r;
    // q . mu for this row, from the BF16 row in global memory (128-key instance)
    float qmu = 0.0f;
    if (!kMuRows && warp < 4 && qrow < N) {
      const uint4* qr = reinterpret_cast<const uint4*>(p.q + (hbase + qrow) * 128);
      const float* mu = p.k_mean + (size_t)head * 128;
#pragma unroll 4
      for (int c = 0; c < 16; ++c) {
        const uint4 raw = __ldg(qr + c);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          qmu = fmaf(f.x, __ldg(mu + 8 * c + 2 * e), qmu);
          qmu = fmaf(f.y, __ldg(mu + 8 * c + 2 * e + 1), qmu);
        }
      }
    }
    float m2 = -INFINITY, l2 = 0.0f;
    for (int ch = 0; ch < nch; ++ch) {
      if (nch > 1) gather(ch);
      const int nk = min(kKeys, kc - kKeys * ch);
      if (warp == kCorrIssuer) {
        if (lane == 0) {
          if (ch == 0) {
            ok = mbar_wait(barQ, ph_q, abort_flag, p.status);
            ph_q ^= 1u;
          }
          if (ok) {
            tc_fence_after();
            const uint64_t dQ = make_sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dK = make_sdesc_sw128(smem_u32(sK), 16, 1024);
#pragma unroll
            for (int k = 0; k < 8; ++k) {           // 16 channels per MMA
              const uint64_t oq = (uint64_t)((k >> 2) * (16384 >> 4) + (k & 3) * 2);
              const uint64_t ok2 = (uint64_t)((k >> 2) * (T::kKVHalf >> 4) + (k & 3) * 2);
              mma_bf16_ss(tmem, dQ + oq, dK + ok2, T::kIdescS, k > 0);
            }
            tc_commit(barS);
            if (ch == nch - 1 && tq + (int)gridDim.x < ntq) {
              // sQ is free once this S completed: load the next tile's Q
              if (mbar_wait(barS, ph_s, abort_flag, p.status)) {
                mbar_arrive_expect_tx(barQ, T::kQBytes);
                tma_load_3d(sQ, &tmQ, barQ, 0, (tq + (int)gridDim.x) * 128, head);
                tma_load_3d(sQ + 16384, &tmQ, barQ, 64, (tq + (int)gridDim.x) * 128, head);
              } else {
                ok = false;
              }
            }
          }
        }
        __syncwarp();
      } else {
        // ---- row threads: softmax of this chunk
        ok = __all_sync(0xffffffffu, mbar_wait(barS, ph_s, abort_flag, p.status));
        tc_fence_after();
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        float x[kKeys];
        uint32_t u[kKeys];
#pragma unroll
        for (int c = 0; c < kKeys / 32; ++c) tmem_ld32(tmem + lane_off + 32u * c, *reinterpret_cast<uint32_t(*)[32]>(&u[32 * c]));
        tmem_wait_ld();
        if constexpr (kMuRows)
          qmu = (__uint_as_float(u[kKeys - 3]) + __uint_as_float(u[kKeys - 2])) + __uint_as_float(u[kKeys - 1]);
#pragma unroll
        for (int e = 0; e < kKeys; ++e)
          x[e] = (e < nk) ? (__uint_as_float(u[e]) - qmu) * c_log2e : -INFINITY;
        float tmax = x[0];
#pragma unroll
        for (int e = 1; e < kKeys; ++e) tmax = fmaxf(tmax, x[e]);
        const float m_new = fmaxf(m2, tmax);
        const float alpha = m2 == -INFINITY ? 0.0f : ex2_approx(m2 - m_new);
        float ls = 0.0f;
#pragma unroll
        for (int c8 = 0; c8 < kKeys / 8; ++c8) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float pa = ex2_approx(x[8 * c8 + 2 * e] - m_new);
            const float pb = ex2_approx(x[8 * c8 + 2 * e + 1] - m_new);
            ls += pa + pb;
            const __nv_bfloat162 h = __floats2bfloat162_rn(pa, pb);
            const float2 hf = __bfloat1622float2(h);
            const __nv_bfloat162 lo = __floats2bfloat162_rn(pa - hf.x, pb - hf.y);
            hw[e] = *reinterpret_cast<const uint32_t*>(&h);
            lw[e] = *reinterpret_cast<const uint32_t*>(&lo);
          }
          const uint32_t off = tile_chunk_off(r, c8, 16384);
          *reinterpret_cast<uint4*>(sPhi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(sPlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        if (ch > 0) {
          // O holds the previous chunks' P.V: rescale when the maximum moved
          ok = ok && __all_sync(0xffffffffu, mbar_wait(barPV, ph_pv ^ 1u, abort_flag, p.status));
          tc_fence_after();
          if (__any_sync(0xffffffffu, m_new != m2)) {
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t o[32];
              tmem_ld32(tmem + 128u + lane_off + 32u * c, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tmem + 128u + lane_off + 32u * c, o);
            }
            tmem_wait_st();
          }
        }
        l2 = l2 * alpha + ls;
        m2 = m_new;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(barP);
      }
      ph_s ^= 1u;
      if (warp == kCorrIssuer) {
        if (lane == 0 && ok) {
          ok = mbar_wait(barP, ph_p, abort_flag, p.status);
          if (ok) {
            tc_fence_after();
            const uint64_t dPh = make_sdesc_sw128(smem_u32(sPhi), 16, 1024);
            const uint64_t dPl = make_sdesc_sw128(smem_u32(sPlo), 16, 1024);
            const uint64_t dV = make_sdesc_sw128(smem_u32(sV), T::kKVHalf, 1024);
#pragma unroll
            for (int k = 0; k < kKeys / 16; ++k) {  // 16 keys per MMA
              const uint64_t offp = (uint64_t)((k >> 2) * (16384 >> 4) + (k & 3) * 2);
              mma_bf16_ss(tmem + 128u, dPh + offp, dV + 128u * k, T::kIdescPV, ch > 0 || k > 0);
              mma_bf16_ss(tmem + 128u, dPl + offp, dV + 128u * k, T::kIdescPV, 1);
            }
          }
          tc_commit(barPV);                    // also on the error path: O settles
        }
        __syncwarp();
      }
      ph_p ^= 1u;
      ph_pv ^= 1u;
      if (nch > 1) {
        // the next chunk's gather overwrites sK / sV: wait for this PV
        if (warp < 4) ok = ok && __all_sync(0xffffffffu, mbar_wait(barPV, ph_pv ^ 1u, abort_flag, p.status));
        __syncthreads();
      }
    }
    // ---- epilogue: merge with the FP8 part and write this row
    if (warp < 4) {
      ok = ok && __all_sync(0xffffffffu, mbar_wait(barPV, ph_pv ^ 1u, abort_flag, p.status));
      tc_fence_after();
      const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
      const bool store = qrow < N && ok;
      float w1 = 0.0f, w2 = 0.0f, inv = 0.0f, l1 = 0.0f;
      if (store) {
        const float2 st = p.stats[hbase + qrow];
        l1 = st.y;
        const float M = fmaxf(st.x, m2);
        w1 = l1 > 0.0f ? ex2_approx(st.x - M) : 0.0f;
        w2 = ex2_approx(m2 - M);
        const float L = l1 * w1 + l2 * w2;
        inv = L > 0.0f ? 1.0f / L : 0.0f;
      }
      const float a1 = (p.o1_raw ? w1 : l1 * w1) * inv, a2 = w2 * inv;
      // the FP8 part's rows come in through shared memory (the P buffers are
      // free once PV completed): the warp loads its 32 rows 32 columns at a
      // time with coalesced 16-byte accesses (8 lanes per 128-byte row
      // segment), then each thread reads its own row; two staging buffers let
      // the next chunk's loads fly while this one is merged
      const int wrow0 = tq * 128 + 32 * warp;
      uint8_t* stg_buf[2] = {sPhi + warp * 4096, sPlo + warp * 4096};
      float4 nxt[8];
      auto load_chunk = [&](int c) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int grow = wrow0 + 4 * i + (lane >> 3);
          nxt[i] = (ok && grow < N)
                       ? __ldg(reinterpret_cast<const float4*>(p.o1 + (hbase + (size_t)grow) * 128 + 32 * c) + (lane & 7))
                       : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
      };
      load_chunk(0);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint8_t* stg = stg_buf[c & 1];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + (lane >> 3), q = lane & 7;
          *reinterpret_cast<float4*>(stg + rr * 128 + ((q ^ (rr & 7)) << 4)) = nxt[i];
        }
        if (c + 1 < 4) load_chunk(c + 1);          // in flight during this chunk's merge
        __syncwarp();
        float4 f1[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) f1[q] = *reinterpret_cast<const float4*>(stg + lane * 128 + ((q ^ (lane & 7)) << 4));
        uint32_t o[32];
        tmem_ld32(tmem + 128u + lane_off + 32u * c, o);
        tmem_wait_ld();
        if (!store) continue;
        float res[32];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float4 f = f1[e];
          res[4 * e] = f.x * a1 + __uint_as_float(o[4 * e]) * a2;
          res[4 * e + 1] = f.y * a1 + __uint_as_float(o[4 * e + 1]) * a2;
          res[4 * e + 2] = f.z * a1 + __uint_as_float(o[4 * e + 2]) * a2;
          res[4 * e + 3] = f.w * a1 + __uint_as_float(o[4 * e + 3]) * a2;
        }
        const size_t orow = hbase + qrow;
        if (p.out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * 128 + 32 * c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(res[4 * e], res[4 * e + 1], res[4 * e + 2], res[4 * e + 3]);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow * 128 + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t w4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(res[8 * e + 2 * u], res[8 * e + 2 * u + 1]);
              w4[u] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            dst[e] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
      tc_fence_before();
    }
    __syncthreads();                            // Q, P and TMEM free for the next tile
    if (!__syncthreads_and(ok)) break;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kCorrIssuer) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace fqa
