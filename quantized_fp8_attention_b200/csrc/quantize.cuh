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
//   amax   = max |x| over the block's (at most 64) x 128 values;
//   s      = amax / 448, inv = 448 / amax (RN divisions; 0 and 0 if amax = 0);
//   code   = E4M3_RNE_satfinite(fl32(x * inv))   (x / s where inv overflows,
//            signed zeros where s underflows);
//   sv_max = max over the head's V block scales.
// Any N >= 1: the last block of a head holds the N - 64*(ceil(N/64)-1)
// remaining tokens, and its scale is their absmax alone.
// Inputs are BF16 [B,H,N,128]; codes are written in the same layout.
#pragma once

#include <type_traits>

#include "device.cuh"

namespace fqa {

// ---------------------------------------------------------------------------
// Fused quantizer: one cooperative persistent launch in three phases separated
// by grid barriers (the K codes need the K mean, which needs all of K):
//   1   V units -> codes and scales; then K units -> per-unit partial sums
//       (per channel, 64 tokens in order), K marked evict-last in L2 for 3
//   2   per (b, h): k_mean from the partials in block order; sv_max = max of
//       the V unit scales (no atomics)
//   3   K units -> smoothed codes and scales, newest units of 1 first (each
//       unit's head mean row arrives with the unit)
// Q is needed by none of the phases, so its units fill the barrier waits:
// each barrier is split into an arrival and a wait, and the first half of
// the Q units runs between the arrival and the wait of barrier 1, the second
// half between those of barrier 2 (while other SMs finish their K units, and
// while phase 2 runs), keeping HBM busy through both.
// Unit u = (b*H + h)*ceil(N/64) + j is one 64-token block of one head: 16 KB
// of contiguous BF16 per tensor (the last block of a head may be shorter).  Units are handed out through work queues
// (counters the launch zeroes), so the SMs that stream faster take more.
// All loads are 1-D bulk copies into a shared-memory ring of kRingBytes, cut
// into as many slots as the phase's unit size allows, so each SM keeps several
// units in flight.  Thread t handles the 16-byte chunks t, t+T, t+2T, ... of
// a unit (T threads, 8 channels a chunk).  Every wait is bounded.

constexpr int kQuantThreads = 256;
constexpr int kQuantWarps = kQuantThreads / 32;
constexpr int kBlockBytes = kQBlock * kHeadDim * 2;            // 16 KB of BF16
constexpr int kChunks = kBlockBytes / 16 / kQuantThreads;       // 16-byte chunks per thread
constexpr int kVals = 8 * kChunks;
constexpr int kRingBytes = 48 * 1024;             // four CTAs per SM
constexpr int kMaxSlots = kRingBytes / kBlockBytes;
constexpr int kSideBytes = kHeadDim * 4;           // per slot: a head's k_mean row (phase 3)
constexpr int kQuantSmem = kRingBytes + kMaxSlots * kSideBytes + 128;
constexpr int kPartialRowsPerSlot = kBlockBytes / (kHeadDim * 4);   // 32 partial rows per 16 KB
// CTAs the shared memory admits per SM (the register cap follows from it)
constexpr int kQuantMinCtas = (228 * 1024) / (kQuantSmem + 2048) < 1 ? 1 : (228 * 1024) / (kQuantSmem + 2048);
static_assert(kMaxSlots >= 3 && kMaxSlots <= 32, "ring size");
static_assert(kQuantThreads >= 2 * kHeadDim, "k_mean and sv_max threads");
static_assert((kQuantThreads * 8) % kHeadDim == 0, "chunk c of thread t starts at channel 8t mod 128");

// Counters the launch zeroes (in the workspace, after the partial sums).
constexpr int kCtrBarrier = 0;     // grid barrier arrivals
constexpr int kCtrV = 1;           // next V unit (phase 1)
constexpr int kCtrK = 2;           // next K unit of phase 1
constexpr int kCtrK3 = 3;          // next unit of phase 3 (counted from the end)
constexpr int kCtrQA = 4;          // next Q unit of the first half
constexpr int kCtrQB = 5;          // next Q unit of the second half
constexpr int kNumCtr = 6;

// Grid barrier, split: grid_arrive() publishes this CTA's earlier writes and
// counts it in; grid_wait(round) waits until every CTA of the grid has
// arrived `round` times (round 1, 2, ...), giving up after kWaitLimitNs.
// Work between the two calls is not covered by the barrier.
__device__ __forceinline__ void grid_arrive(unsigned int* ctr) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
  }
}
__device__ __forceinline__ bool grid_wait(unsigned int* ctr, unsigned int round, uint32_t* status,
                                          volatile int* failed) {
  if (threadIdx.x == 0) {
    const unsigned int target = round * gridDim.x;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      unsigned int v = *reinterpret_cast<volatile unsigned int*>(ctr);
      if ((int)(v - target) >= 0) break;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        atomicOr(status, kStatusTimeout);
        *failed = 1;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
    // what other CTAs wrote before the barrier is read next by bulk copies
    asm volatile("fence.proxy.async.global;" ::: "memory");
  }
  __syncthreads();
  return *failed == 0;
}

// The values of this thread's chunks of a staged BF16 unit; chunks at or
// beyond nvalid (past a short block's tokens) read as zeros.
__device__ __forceinline__ void chunks_to_f32(const uint8_t* blk, int nvalid, float (&x)[kVals]) {
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    const int c = threadIdx.x + kQuantThreads * i;
    const uint4 raw = c < nvalid ? *reinterpret_cast<const uint4*>(blk + 16 * c) : make_uint4(0, 0, 0, 0);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h2[e]);
      x[i * 8 + 2 * e] = f.x;
      x[i * 8 + 2 * e + 1] = f.y;
    }
  }
}

// Residual squares of one chunk (8 consecutive channels): the sequential
// binary32 sum of fl32(r^2), r = fl32(x - fl32(dec(code) * scale)), for the
// four packed code pairs w[0..3] (element 2e in bits [0,8) of w[e]).
__device__ __forceinline__ float residual_sq8(const float* x, const uint32_t (&w)[4], float scale) {
  float acc = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 d = e4m3x2_to_f2(w[e]);
    const float r0 = __fsub_rn(x[2 * e], __fmul_rn(d.x, scale));
    const float r1 = __fsub_rn(x[2 * e + 1], __fmul_rn(d.y, scale));
    acc = __fadd_rn(acc, __fmul_rn(r0, r0));
    acc = __fadd_rn(acc, __fmul_rn(r1, r1));
  }
  return acc;
}

// Lane-wise max(|a|, |b|) of two BF16 pairs: max.xorsign.abs leaves that
// magnitude in each lane (the sign bit, an XOR of the inputs', is not used),
// so a tree of them ends with the largest magnitude of each lane.
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// BF16 pair (element 0 in the low half) -> its two exact binary32 values.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// The largest |x| over the CTA, from this thread's m >= 0 (red: one float
// per warp, in buffer `slot`; non-negative binary32 values order like their
// bit patterns, so the warp maximum is an integer reduction), and the block's
// scale and inverse.  The CTA-wide sync also combines `ok` (this thread's
// wait for the unit): unless every thread's is true, false is returned.  It
// is the unit's one sync: the caller's slot may be refilled after it and the
// other `red` buffer is free for the next unit.
__device__ __forceinline__ bool block_scale(float m, float* red, int slot, bool ok, float& scale,
                                            float& inv) {
  const int t = threadIdx.x;
  const uint32_t mw = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  if ((t & 31) == 0) red[slot * kQuantWarps + (t >> 5)] = __uint_as_float(mw);
  if (!__syncthreads_and(ok)) return false;
  static_assert(kQuantWarps == 8, "two float4 loads per buffer");
  const float4 r0 = *reinterpret_cast<const float4*>(red + slot * kQuantWarps);
  const float4 r1 = *reinterpret_cast<const float4*>(red + slot * kQuantWarps + 4);
  const float a = fmax3(fmax3(r0.x, r0.y, r0.z), fmax3(r0.w, r1.x, r1.y), fmaxf(r1.z, r1.w));
  scale = a > 0.0f ? __fdiv_rn(a, 448.0f) : 0.0f;
  inv = a > 0.0f ? __fdiv_rn(448.0f, a) : 0.0f;
  if (scale == 0.0f) inv = 0.0f;               // amax / 448 underflowed: flush the block
  return true;
}

// Codes of 8 values (one chunk) -> two words, value 0 in bits [0,8): x * inv,
// or x / scale where inv overflowed (amax below about 1.3e-36, block-uniform:
// the block's zeros then stay zeros instead of 0 * inf).
__device__ __forceinline__ uint2 chunk_codes(const float (&x)[8], float scale, float inv) {
  if (isinf(inv)) {
    return make_uint2(e4m3x4(__fdiv_rn(x[0], scale), __fdiv_rn(x[1], scale), __fdiv_rn(x[2], scale),
                             __fdiv_rn(x[3], scale)),
                      e4m3x4(__fdiv_rn(x[4], scale), __fdiv_rn(x[5], scale), __fdiv_rn(x[6], scale),
                             __fdiv_rn(x[7], scale)));
  }
  const float2 i2 = make_float2(inv, inv);
  const float2 p0 = f2_mul(make_float2(x[0], x[1]), i2), p1 = f2_mul(make_float2(x[2], x[3]), i2);
  const float2 p2 = f2_mul(make_float2(x[4], x[5]), i2), p3 = f2_mul(make_float2(x[6], x[7]), i2);
  return make_uint2(e4m3x4(p0.x, p0.y, p1.x, p1.y), e4m3x4(p2.x, p2.y, p3.x, p3.y));
}

// Block absmax, scale and the codes of this thread's chunks of a staged BF16
// unit (raw: the chunks as loaded; chunks at or beyond nvalid are zeros and
// are not stored; chunk c's 8 codes go to byte 8c of dst).  The absmax is
// taken on the BF16 pairs (BF16 -> binary32 is exact, so it is the binary32
// absmax); the values are converted after the sync.
__device__ __forceinline__ bool quantize_chunks_bf16(const uint4 (&raw)[kChunks], float* red, uint8_t* dst,
                                                     int slot, int nvalid, uint64_t policy, bool ok,
                                                     float& scale_out) {
  const int t = threadIdx.x;
  static_assert(kChunks == 4, "a 16-word tree");
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    w[4 * i + 0] = bf16x2_absmax(raw[i].x, raw[i + 2].x);
    w[4 * i + 1] = bf16x2_absmax(raw[i].y, raw[i + 2].y);
    w[4 * i + 2] = bf16x2_absmax(raw[i].z, raw[i + 2].z);
    w[4 * i + 3] = bf16x2_absmax(raw[i].w, raw[i + 2].w);
  }
  const uint32_t w4 = bf16x2_absmax(bf16x2_absmax(w[0], w[4]), bf16x2_absmax(w[1], w[5]));
  const uint32_t w5 = bf16x2_absmax(bf16x2_absmax(w[2], w[6]), bf16x2_absmax(w[3], w[7]));
  const float2 mf = bf16x2_to_f2(bf16x2_absmax(w4, w5));
  float scale, inv;
  if (!block_scale(fmaxf(fabsf(mf.x), fabsf(mf.y)), red, slot, ok, scale, inv)) return false;
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    float x[8];
    const uint32_t ww[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = bf16x2_to_f2(ww[e]);
      x[2 * e] = f.x;
      x[2 * e + 1] = f.y;
    }
    const uint2 c = chunk_codes(x, scale, inv);
    if (t + kQuantThreads * i < nvalid) st_global_v2_hint(dst + 8 * (t + kQuantThreads * i), c.x, c.y, policy);
  }
  scale_out = scale;
  return true;
}

// The same for binary32 values x (this thread's chunks, chunk i in x[8i..8i+8);
// values of chunks past nvalid must be zeros).  rsq (optional): each chunk's
// residual squares (residual_sq8).
__device__ __forceinline__ bool quantize_chunks(const float (&x)[kVals], float* red, uint8_t* dst, int slot,
                                                int nvalid, uint64_t policy, bool ok, float& scale_out,
                                                float* rsq = nullptr) {
  const int t = threadIdx.x;
  static_assert(kVals == 32, "a 32-value tree");
  float m[11];
#pragma unroll
  for (int i = 0; i < 10; ++i) m[i] = fmax3(fabsf(x[3 * i]), fabsf(x[3 * i + 1]), fabsf(x[3 * i + 2]));
  m[10] = fmaxf(fabsf(x[30]), fabsf(x[31]));
  const float m0 = fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmax3(m[6], m[7], m[8]));
  float scale, inv;
  if (!block_scale(fmax3(m0, m[9], m[10]), red, slot, ok, scale, inv)) return false;
#pragma unroll
  for (int i = 0; i < kChunks; ++i) {
    const float(&xc)[8] = *reinterpret_cast<const float(*)[8]>(&x[8 * i]);
    const uint2 c = chunk_codes(xc, scale, inv);
    if (t + kQuantThreads * i < nvalid) st_global_v2_hint(dst + 8 * (t + kQuantThreads * i), c.x, c.y, policy);
    if (rsq) {
      const uint32_t w[4] = {c.x & 0xFFFFu, c.x >> 16, c.y & 0xFFFFu, c.y >> 16};
      rsq[i] = residual_sq8(&x[8 * i], w, scale);
    }
  }
  scale_out = scale;
  return true;
}

__global__ void __launch_bounds__(kQuantThreads, kQuantMinCtas) quantize_fused_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, uint8_t* __restrict__ q8, uint8_t* __restrict__ k8,
    uint8_t* __restrict__ v8, float* __restrict__ sq, float* __restrict__ sk,
    float* __restrict__ sv, float* __restrict__ sv_max, float* __restrict__ k_mean,
    float* __restrict__ partial, unsigned int* __restrict__ ctr, int B, int H, int N,
    uint32_t* status, float* __restrict__ k_err, int in_P) {
  extern __shared__ uint8_t qsmem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsmem_raw) + 127) & ~uintptr_t(127));
  uint8_t* side = ring + kRingBytes;               // kMaxSlots x kSideBytes
  __shared__ uint64_t full[kMaxSlots];
  __shared__ int slot_unit[kMaxSlots];
  __shared__ __align__(16) float red[2 * kQuantWarps];
  __shared__ int failed, abort_flag;
  const int t = threadIdx.x;
  const int nblk = (N + kQBlock - 1) / kQBlock;
  const int nunits = B * H * nblk;
  const int G = gridDim.x;
  if (t == 0) {
    failed = 0;
    abort_flag = 0;
    for (int s = 0; s < kMaxSlots; ++s) mbar_init(&full[s], 1);
    mbar_fence_init();
  }
  __syncthreads();
  const uint64_t pol_first = l2_policy_evict_first();
  const uint64_t pol_last = l2_policy_evict_last();
  uint32_t phase_bits = 0;                         // parity of each ring barrier

  // One pipelined pass with slots of slot_bytes.  next() (thread 0) yields
  // the next unit index, or -1 when there is none and from then on;
  // issue(u, dst, bar) starts unit u's bulk copies (it arms bar itself);
  // body(u, slot memory, ok, parity) runs on all threads, in the order next()
  // gave the units, ok being this thread's wait for the unit and parity the
  // unit's count mod 2.  A body that returns bool contains one
  // __syncthreads_and(ok) after its last read of the slot (the slot is then
  // refilled while the body finishes) and returns its result; any other body
  // is fenced by syncs on both sides.  Every started copy is waited for
  // before the pass returns, unless a wait timed out (returns false).
  auto run = [&](int slot_bytes, auto next, auto issue, auto body) -> bool {
    const int nslots = kRingBytes / slot_bytes;
    // every thread has left the previous pass (a body-synced pass ends with
    // threads past their last sync but not yet at the loop's exit test)
    __syncthreads();
    if (t == 0)
      for (int s = 0; s < nslots - 1; ++s) {
        const int u = next();
        slot_unit[s] = u;
        if (u >= 0) issue(u, ring + s * slot_bytes, &full[s]);
      }
    __syncthreads();
    int it = 0;
    for (int s = 0;; s = (s + 1 == nslots) ? 0 : s + 1) {
      const int u = slot_unit[s];
      if (u < 0) break;                            // CTA-uniform
      if (t == 0) {
        // the slot before s was released by the barrier that ended its unit
        const int s2 = (s == 0) ? nslots - 1 : s - 1;
        const int u2 = next();
        slot_unit[s2] = u2;
        if (u2 >= 0) issue(u2, ring + s2 * slot_bytes, &full[s2]);
      }
      const bool ok = mbar_wait(&full[s], (phase_bits >> s) & 1u, &abort_flag, status);
      phase_bits ^= 1u << s;
      using R = decltype(body(u, ring, ok, 0));
      if constexpr (std::is_same<R, bool>::value) {
        if (!body(u, ring + s * slot_bytes, ok, it & 1)) return false;
      } else {
        if (!__syncthreads_and(ok)) return false;
        body(u, ring + s * slot_bytes, ok, it & 1);
        __syncthreads();                           // slot s and slot_unit free again
      }
      ++it;
    }
    return true;
  };
  // a shared work queue over units [lo, hi): ctr[c] counts the units handed out
  auto queue = [&](int c, int lo, int hi, bool reverse) {
    bool drained = false;
    return [=]() mutable -> int {
      if (drained) return -1;
      const unsigned int i = atomicAdd(&ctr[c], 1u);
      if (i >= (unsigned int)(hi - lo)) {
        drained = true;
        return -1;
      }
      return reverse ? hi - 1 - (int)i : lo + (int)i;
    };
  };
  // element offset of unit u in a [B,H,N,128] tensor (the codes, and the
  // inputs when in_P == 1), and its token count
  auto unit_off = [&](int u) {
    const int hd = u / nblk;
    return ((size_t)hd * N + (size_t)(u - hd * nblk) * kQBlock) * kHeadDim;
  };
  // element offset of unit u in the inputs: with in_P > 1 they are in the
  // sequence all-to-all layout [B, in_P, H, N / in_P, 128] (chunk p holds
  // tokens [p N/in_P, (p+1) N/in_P) of every head; N / in_P is a multiple of
  // 64, so no block straddles two chunks)
  const int nl = N / in_P;
  auto unit_in = [&](int u) -> size_t {
    if (in_P == 1) return unit_off(u);
    const int hd = u / nblk;
    const int n0 = (u - hd * nblk) * kQBlock, c = n0 / nl;
    const int b = hd / H, h = hd - b * H;
    return ((((size_t)b * in_P + c) * H + h) * nl + (n0 - c * nl)) * kHeadDim;
  };
  auto unit_rows = [&](int u) { return min(kQBlock, N - (u % nblk) * kQBlock); };

  // Q or V units (streamed once: evict-first) -> codes and block scales
  auto pass_qv = [&](const __nv_bfloat16* src, uint8_t* codes, float* scales, auto next) -> bool {
    return run(kBlockBytes, next,
        [&](int u, uint8_t* dst, uint64_t* bar) {
          const uint32_t bytes = (uint32_t)unit_rows(u) * kHeadDim * 2;
          mbar_arrive_expect_tx(bar, bytes);
          bulk_load(dst, src + unit_in(u), bytes, bar, pol_first);
        },
        [&](int u, const uint8_t* blk, bool ok, int par) -> bool {
          const int nvalid = unit_rows(u) * (kHeadDim * 2 / 16);
          uint4 raw[kChunks];
#pragma unroll
          for (int i = 0; i < kChunks; ++i) {
            const int c = t + kQuantThreads * i;
            raw[i] = c < nvalid ? *reinterpret_cast<const uint4*>(blk + 16 * c) : make_uint4(0, 0, 0, 0);
          }
          float sc;
          if (!quantize_chunks_bf16(raw, red, codes + unit_off(u), par, nvalid, pol_first, ok, sc)) return false;
          if (t == 0) scales[u] = sc;
          return true;
        });
  };
  const int nqa = (nunits + 1) / 2;                // Q units before barrier 1's wait

  // ---- phase 1: V, then the K partial sums (one thread per channel adds the
  // unit's 64 tokens in order); K stays in L2 for phase 3
  bool ok = pass_qv(v, v8, sv, queue(kCtrV, 0, nunits, false));
  if (ok)
    ok = run(kBlockBytes, queue(kCtrK, 0, nunits, false),
        [&](int u, uint8_t* dst, uint64_t* bar) {
          const uint32_t bytes = (uint32_t)unit_rows(u) * kHeadDim * 2;
          mbar_arrive_expect_tx(bar, bytes);
          bulk_load(dst, k + unit_in(u), bytes, bar, pol_last);
        },
        [&](int u, const uint8_t* blk, bool, int) {
          if (t < kHeadDim) {
            const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(blk);
            const int rows = unit_rows(u);
            float acc = 0.0f;
            if (rows == kQBlock) {
#pragma unroll 16
              for (int n = 0; n < kQBlock; ++n) acc = __fadd_rn(acc, __bfloat162float(kb[n * kHeadDim + t]));
            } else {
              for (int n = 0; n < rows; ++n) acc = __fadd_rn(acc, __bfloat162float(kb[n * kHeadDim + t]));
            }
            partial[(size_t)u * kHeadDim + t] = acc;
          }
        });
  if (!ok) failed = 1;
  grid_arrive(&ctr[kCtrBarrier]);
  // the first half of Q while the other SMs finish phase 1
  if (ok && !pass_qv(q, q8, sq, queue(kCtrQA, 0, nqa, false))) failed = 1;
  if (!grid_wait(&ctr[kCtrBarrier], 1, status, &failed)) return;

  // ---- phase 2: per (b, h), k_mean (threads 0..127: one channel each, the
  // partials staged 32 rows a slot and added in block order) and sv_max
  // (threads 128..255: a max over the V unit scales, any order; the scales
  // come from other SMs, so the loads bypass L1)
  for (int hd = blockIdx.x; hd < B * H; hd += G) {
    if (t >= kHeadDim && t < 2 * kHeadDim) {
      float m = 0.0f;
      for (int j = t - kHeadDim; j < nblk; j += kHeadDim) m = fmaxf(m, __ldcg(sv + (size_t)hd * nblk + j));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if ((t & 31) == 0) red[kQuantWarps + ((t - kHeadDim) >> 5)] = m;
    }
    const float* src = partial + (size_t)hd * nblk * kHeadDim;
    const int nchunk = (nblk + kPartialRowsPerSlot - 1) / kPartialRowsPerSlot;
    int next_chunk = 0;
    float acc = 0.0f;
    ok = run(kBlockBytes, [&]() -> int { return next_chunk < nchunk ? next_chunk++ : -1; },
        [&](int i, uint8_t* dst, uint64_t* bar) {
          const int rows = min(kPartialRowsPerSlot, nblk - i * kPartialRowsPerSlot);
          mbar_arrive_expect_tx(bar, rows * kHeadDim * 4);
          bulk_load(dst, src + (size_t)i * kPartialRowsPerSlot * kHeadDim, rows * kHeadDim * 4, bar,
                    pol_first);
        },
        [&](int i, const uint8_t* blk, bool, int) {
          if (t < kHeadDim) {
            const float* pr = reinterpret_cast<const float*>(blk);
            const int rows = min(kPartialRowsPerSlot, nblk - i * kPartialRowsPerSlot);
#pragma unroll 8
            for (int r = 0; r < rows; ++r) acc = __fadd_rn(acc, pr[r * kHeadDim + t]);
          }
        });
    if (!ok) {
      failed = 1;
      break;
    }
    if (t < kHeadDim) k_mean[(size_t)hd * kHeadDim + t] = __fdiv_rn(acc, (float)N);
    if (t == kHeadDim) {
      float m = red[kQuantWarps];
#pragma unroll
      for (int w = 1; w < kHeadDim / 32; ++w) m = fmaxf(m, red[kQuantWarps + w]);
      sv_max[hd] = m;
    }
    __syncthreads();                               // red reused by the next head
  }
  grid_arrive(&ctr[kCtrBarrier]);
  // the second half of Q while phase 2 completes on the other SMs
  if (!failed && !pass_qv(q, q8, sq, queue(kCtrQB, nqa, nunits, false))) failed = 1;
  if (!grid_wait(&ctr[kCtrBarrier], 2, status, &failed)) return;

  // ---- phase 3: K codes, newest units of phase 1 first.  Each unit's head
  // k_mean row (512 B) arrives with it, in the slot's side buffer.
  run(kBlockBytes, queue(kCtrK3, 0, nunits, true),
      [&](int u, uint8_t* dst, uint64_t* bar) {
        const uint32_t bytes = (uint32_t)unit_rows(u) * kHeadDim * 2;
        mbar_arrive_expect_tx(bar, bytes + kSideBytes);
        bulk_load(dst, k + unit_in(u), bytes, bar, pol_first);
        // (the row is read again by every unit of its head: it stays in L2)
        bulk_load(side + (dst - ring) / kBlockBytes * kSideBytes, k_mean + (size_t)(u / nblk) * kHeadDim,
                  kSideBytes, bar, pol_last);
      },
      [&](int u, const uint8_t* blk, bool ok, int par) -> bool {
        // every chunk of this thread starts at channel 8t mod 128
        const float* mu = reinterpret_cast<const float*>(side + (blk - ring) / kBlockBytes * kSideBytes) +
                          ((8 * t) & (kHeadDim - 1));
        // x - mu as x + (-mu): the same IEEE result, two channels per add
        float2 nmu[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) nmu[e] = make_float2(-mu[2 * e], -mu[2 * e + 1]);
        const int nvalid = unit_rows(u) * (kHeadDim * 2 / 16);
        float x[kVals];
        chunks_to_f32(blk, nvalid, x);
#pragma unroll
        for (int i4 = 0; i4 < kChunks; ++i4) {
          // chunks past a short block's tokens stay 0: they must not enter amax
          if (t + kQuantThreads * i4 < nvalid) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 d = f2_add(make_float2(x[8 * i4 + 2 * e], x[8 * i4 + 2 * e + 1]), nmu[e]);
              x[8 * i4 + 2 * e] = d.x;
              x[8 * i4 + 2 * e + 1] = d.y;
            }
          }
        }
        float s_k;
        if (k_err == nullptr) {
          if (!quantize_chunks(x, red, k8 + unit_off(u), par, nvalid, pol_first, ok, s_k)) return false;
          if (t == 0) sk[u] = s_k;
          return true;
        }
        // with the per-key quantization error: chunk i of this thread is
        // channels 8 (t % 16) .. +8 of token t / 16 + 16 i of the unit; the 16
        // lanes of a token combine their chunk sums pairwise in the pinned
        // order g_l + g_l^8, then ^4, ^2, ^1 (identical in every lane)
        float rsq[kChunks];
        if (!quantize_chunks(x, red, k8 + unit_off(u), par, nvalid, pol_first, ok, s_k, rsq)) return false;
        if (t == 0) sk[u] = s_k;
        const size_t tok0 = unit_off(u) / kHeadDim;
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
          float e = rsq[i];
          e = __fadd_rn(e, __shfl_xor_sync(0xffffffffu, e, 8));
          e = __fadd_rn(e, __shfl_xor_sync(0xffffffffu, e, 4));
          e = __fadd_rn(e, __shfl_xor_sync(0xffffffffu, e, 2));
          e = __fadd_rn(e, __shfl_xor_sync(0xffffffffu, e, 1));
          const int c = t + kQuantThreads * i;
          if ((t & 15) == 0 && c < nvalid) k_err[tok0 + c / 16] = e;
        }
        return true;
      });
}

// Exercises the bounded-wait path: one thread waits on an mbarrier that no
// one arrives on; after limit_ns the wait gives up, sets the timeout bit of
// the status word and the kernel returns normally.
__global__ void wait_timeout_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  mbar_init(&bar, 1);
  abort_flag = 0;
  mbar_fence_init();
  mbar_wait_limit(&bar, 0, &abort_flag, status, limit_ns);
}

// The exponential every attention kernel uses (ex2.approx.ftz.f32) at every
// binary32 x in [lo, hi] (lo <= hi <= 0 here), against binary64 exp2: the
// largest relative error, as its bit pattern (non-negative floats order like
// their bits), into *max_rel_bits.
__global__ void exp2_error_kernel(uint32_t lo_bits, uint32_t n, unsigned int* max_rel_bits) {
  float worst = 0.0f;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    // negative floats: larger magnitude <-> larger bit pattern; walk from hi down to lo
    const float x = __uint_as_float(lo_bits - i);
    const float y = ex2_approx(x);
    const double ref = exp2((double)x);
    if (ref >= 0x1p-126) worst = fmaxf(worst, (float)(fabs((double)y - ref) / ref));
  }
  for (int o = 16; o > 0; o >>= 1) worst = fmaxf(worst, __shfl_xor_sync(0xffffffffu, worst, o));
  if ((threadIdx.x & 31) == 0) atomicMax(max_rel_bits, __float_as_uint(worst));
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
