// fqa.cu -- the library's C ABI (include/fqa.h): host-side argument checks,
// TMA tensor-map encoding and kernel launches.  One translation unit holds
// every kernel, so the device status word needs no relocatable device code.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/fqa.h"
#include "attention.cuh"
#include "attention_fp8.cuh"
#include "attention_nvfp4.cuh"
#include "attention_ws.cuh"
#include "correct.cuh"
#include "device.cuh"
#include "quantize.cuh"
#include "quantize_nvfp4.cuh"

namespace fqa {

__device__ uint32_t g_status_word;

constexpr int kMaxDevices = 64;

// Per-device lookups, cached only once they succeed: a failed first call
// (e.g. one made while a stream is being captured) is retried by the next.
struct DeviceCache {
  std::mutex mu;
  uint32_t* status = nullptr;
  int num_sms = 0;
};
DeviceCache g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

static uint32_t* status_ptr(fqa_status* st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *st = FQA_ERR_CUDA;
    return nullptr;
  }
  DeviceCache& c = g_dev[dev];
  std::lock_guard<std::mutex> lock(c.mu);
  if (c.status == nullptr) {
    void* p = nullptr;
    int sms = 0;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        p == nullptr || sms <= 0) {
      *st = FQA_ERR_CUDA;
      return nullptr;
    }
    c.num_sms = sms;
    c.status = static_cast<uint32_t*>(p);
  }
  return c.status;
}

static EncodeTiledFn encoder() {
  std::call_once(g_encode_once, []() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

// 3-D view (channel, row within the head, head) of a [B,H,N,128] tensor; box
// = 128 B of channels x 128 rows x 1 head, 128-byte swizzle.  Rows past N
// (the short last tile of a sequence) are filled with zeros, never read from
// the next head.
static bool make_tmap(CUtensorMap* m, const void* base, bool fp8, int N, int heads) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const uint32_t elt = fp8 ? 1 : 2;
  cuuint64_t dims[3] = {128, (cuuint64_t)N, (cuuint64_t)heads};
  cuuint64_t strides[2] = {128ull * elt, 128ull * elt * (cuuint64_t)N};
  cuuint32_t box[3] = {128u / elt, 128u, 1u};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D view (byte, row within the head, head) of packed E2M1 codes
// [B,H,N,64 B]; box = 64 B x 128 rows x 1 head, 64-byte swizzle (the layout
// the block-scaled MMA reads through a SWIZZLE_64B descriptor).
static bool make_tmap_fp4(CUtensorMap* m, const void* base, int N, int heads) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)N, (cuuint64_t)heads};
  cuuint64_t strides[2] = {64ull, 64ull * (cuuint64_t)N};
  cuuint32_t box[3] = {64u, 128u, 1u};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape checks shared by every call: any N >= 1 (the last 64-token block and
// the last 128-key tile of a head may be short).
static fqa_status check_shape(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1) return FQA_ERR_INVALID_ARG;
  if (d != 128) return FQA_ERR_UNSUPPORTED;
  if (N > 65536) return FQA_ERR_UNSUPPORTED;
  if ((int64_t)B * H > 65535) return FQA_ERR_UNSUPPORTED;
  if ((int64_t)B * H * N >= (int64_t(1) << 31)) return FQA_ERR_UNSUPPORTED;
  return FQA_OK;
}

static fqa_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? FQA_OK : FQA_ERR_CUDA;
}

// SM count of the current device (valid once status_ptr() succeeded on it).
static int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> lock(g_dev[dev].mu);
  return g_dev[dev].num_sms;
}

// BF16: persistent launch, one CTA per SM (or per work item, if fewer).
static fqa_status launch_attention_bf16(const void* q, const void* k, const void* v,
                                        const AttnParams& prm, cudaStream_t stream) {
  const int heads = prm.B * prm.H;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, false, prm.N, heads) || !make_tmap(&tk, k, false, prm.N, heads) ||
      !make_tmap(&tv, v, false, prm.N, heads))
    return FQA_ERR_CUDA;
  if (cudaFuncSetAttribute(attn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           BfTraits::kSmemBytes) != cudaSuccess)
    return FQA_ERR_CUDA;
  const int items = prm.B * prm.H * ((prm.N + kPairRows - 1) / kPairRows);
  const int sms = num_sms();
  if (sms <= 0) return FQA_ERR_CUDA;
  const int grid = items < sms ? items : sms;
  attn_bf16_kernel<<<grid, kWsThreads, BfTraits::kSmemBytes, stream>>>(tq, tk, tv, prm);
  return launch_status();
}

// FP8: persistent launch of the shared-memory-P kernel, one CTA per SM (or
// per work item, if fewer).
static fqa_status launch_attention_fp8(const void* q, const void* k, const void* v,
                                       const AttnParams& prm, cudaStream_t stream) {
  const int heads = prm.B * prm.H;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, true, prm.N, heads) || !make_tmap(&tk, k, true, prm.N, heads) ||
      !make_tmap(&tv, v, true, prm.N, heads))
    return FQA_ERR_CUDA;
  // the instance that carries only what the call needs: the short-tail patch
  // when N is not a multiple of 128, the key mask and row statistics when
  // given
  const bool tail = prm.N % kBlockN != 0;
  const bool masked = prm.kmask != nullptr || prm.row_stats != nullptr;
  using KernelFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const AttnParams);
  KernelFn fn = tail ? (masked ? attn_fp8_kernel<true, true> : attn_fp8_kernel<true, false>)
                     : (masked ? attn_fp8_kernel<false, true> : attn_fp8_kernel<false, false>);
  // a key mask that leaves a key in every 64-key block of an aligned N:
  // patched tiles instead of masking (the caller checks the condition)
  if (prm.patch && !tail && prm.kmask != nullptr) fn = attn_fp8_kernel<false, false, true>;
  if (cudaFuncSetAttribute((const void*)fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           F8Traits::kSmemBytes) != cudaSuccess)
    return FQA_ERR_CUDA;
  const int items = prm.B * prm.H * ((prm.N + 2 * kBlockM - 1) / (2 * kBlockM));
  const int sms = num_sms();
  if (sms <= 0) return FQA_ERR_CUDA;
  const int grid = items < sms ? items : sms;
  fn<<<grid, kF8Threads, F8Traits::kSmemBytes, stream>>>(tq, tk, tv, prm);
  return launch_status();
}

}  // namespace fqa

using namespace fqa;

extern "C" {

int fqa_version(void) { return (1 << 16) | 0; }

const char* fqa_status_string(fqa_status s) {
  switch (s) {
    case FQA_OK: return "FQA_OK";
    case FQA_ERR_INVALID_ARG: return "FQA_ERR_INVALID_ARG";
    case FQA_ERR_UNSUPPORTED: return "FQA_ERR_UNSUPPORTED";
    case FQA_ERR_MISALIGNED: return "FQA_ERR_MISALIGNED";
    case FQA_ERR_CUDA: return "FQA_ERR_CUDA";
    case FQA_ERR_TIMEOUT: return "FQA_ERR_TIMEOUT";
  }
  return "FQA_UNKNOWN_STATUS";
}

// Workspace: the K-mean partial sums [B,H,ceil(N/64),128] FP32, then
// (256-byte aligned) the grid-barrier and work-queue counters of the fused
// quantize launch.
static size_t partial_bytes(int B, int H, int N, int d) {
  return (size_t)B * H * ((N + kQBlock - 1) / kQBlock) * d * sizeof(float);
}

size_t fqa_quantize_workspace_bytes(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d) != FQA_OK) return 0;
  return ((partial_bytes(B, H, N, d) + 255) & ~size_t(255)) + 256;
}

static fqa_status quantize_impl(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                                void* q8, void* k8, void* v8, float* sq, float* sk, float* sv,
                                float* sv_max, float* k_mean, float* k_err, void* workspace,
                                size_t workspace_bytes, void* cuda_stream, int in_P = 1) {
  fqa_status st = check_shape(B, H, N, d);
  if (st != FQA_OK) return st;
  const void* ptrs[] = {q, k, v, q8, k8, v8, sq, sk, sv, sv_max, k_mean, workspace};
  for (const void* p : ptrs)
    if (p == nullptr) return FQA_ERR_INVALID_ARG;
  if (workspace_bytes < fqa_quantize_workspace_bytes(B, H, N, d)) return FQA_ERR_INVALID_ARG;
  const void* a16[] = {q, k, v, q8, k8, v8, k_mean, workspace};   // k_mean: read by bulk copies
  for (const void* p : a16)
    if (!aligned(p, 16)) return FQA_ERR_MISALIGNED;
  const void* a4[] = {sq, sk, sv, sv_max, k_err};
  for (const void* p : a4)
    if (!aligned(p, 4)) return FQA_ERR_MISALIGNED;
  uint32_t* status = status_ptr(&st);
  if (!status) return st;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  float* partial = static_cast<float*>(workspace);
  unsigned int* ctr = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(workspace) +
                                                      ((partial_bytes(B, H, N, d) + 255) & ~size_t(255)));
  const int nunits = B * H * ((N + kQBlock - 1) / kQBlock);
  if (cudaFuncSetAttribute(quantize_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kQuantSmem) != cudaSuccess)
    return FQA_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_fused_kernel, kQuantThreads,
                                                    kQuantSmem) != cudaSuccess ||
      per_sm < 1)
    return FQA_ERR_CUDA;
  int grid = per_sm * num_sms();
  if (grid > nunits) grid = nunits;
  static_assert(kNumCtr * sizeof(unsigned int) <= 256, "counters fit the reserved 256 bytes");
  if (cudaMemsetAsync(ctr, 0, kNumCtr * sizeof(unsigned int), s) != cudaSuccess) return FQA_ERR_CUDA;
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(v);
  uint8_t* q8b = static_cast<uint8_t*>(q8);
  uint8_t* k8b = static_cast<uint8_t*>(k8);
  uint8_t* v8b = static_cast<uint8_t*>(v8);
  void* args[] = {(void*)&qb, (void*)&kb, (void*)&vb, (void*)&q8b, (void*)&k8b, (void*)&v8b,
                  (void*)&sq, (void*)&sk, (void*)&sv, (void*)&sv_max, (void*)&k_mean,
                  (void*)&partial, (void*)&ctr, (void*)&B, (void*)&H, (void*)&N, (void*)&status,
                  (void*)&k_err, (void*)&in_P};
  // cooperative: every CTA is resident, so the grid barriers cannot wait on
  // a CTA that never starts
  if (cudaLaunchCooperativeKernel((const void*)quantize_fused_kernel, dim3(grid), dim3(kQuantThreads),
                                  args, kQuantSmem, s) != cudaSuccess)
    return FQA_ERR_CUDA;
  return launch_status();
}

fqa_status fqa_quantize(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                        void* q8, void* k8, void* v8, float* sq, float* sk, float* sv,
                        float* sv_max, float* k_mean, void* workspace, size_t workspace_bytes,
                        void* cuda_stream) {
  return quantize_impl(q, k, v, B, H, N, d, q8, k8, v8, sq, sk, sv, sv_max, k_mean, nullptr, workspace,
                       workspace_bytes, cuda_stream);
}

fqa_status fqa_quantize_keyerr(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                               void* q8, void* k8, void* v8, float* sq, float* sk, float* sv,
                               float* sv_max, float* k_mean, float* k_err, void* workspace,
                               size_t workspace_bytes, void* cuda_stream) {
  if (k_err == nullptr) return FQA_ERR_INVALID_ARG;
  return quantize_impl(q, k, v, B, H, N, d, q8, k8, v8, sq, sk, sv, sv_max, k_mean, k_err, workspace,
                       workspace_bytes, cuda_stream);
}

static fqa_status check_attention_common(int B, int H, int N, int d, float softmax_scale,
                                         void* out, fqa_out_dtype out_dtype) {
  fqa_status st = check_shape(B, H, N, d);
  if (st != FQA_OK) return st;
  if (!(std::isfinite(softmax_scale) && softmax_scale > 0.0f)) return FQA_ERR_INVALID_ARG;
  if (out == nullptr) return FQA_ERR_INVALID_ARG;
  if (out_dtype != FQA_OUT_BF16 && out_dtype != FQA_OUT_F32) return FQA_ERR_INVALID_ARG;
  if (!aligned(out, 16)) return FQA_ERR_MISALIGNED;
  return FQA_OK;
}

fqa_status fqa_attention_fp8(const void* q8, const void* k8, const void* v8, const float* sq,
                             const float* sk, const float* sv, const float* sv_max, int B, int H,
                             int N, int d, float softmax_scale, void* out,
                             fqa_out_dtype out_dtype, void* cuda_stream) {
  fqa_status st = check_attention_common(B, H, N, d, softmax_scale, out, out_dtype);
  if (st != FQA_OK) return st;
  const void* ptrs[] = {q8, k8, v8, sq, sk, sv, sv_max};
  for (const void* p : ptrs)
    if (p == nullptr) return FQA_ERR_INVALID_ARG;
  const void* a16[] = {q8, k8, v8};
  for (const void* p : a16)
    if (!aligned(p, 16)) return FQA_ERR_MISALIGNED;
  const void* a4[] = {sq, sk, sv, sv_max};
  for (const void* p : a4)
    if (!aligned(p, 4)) return FQA_ERR_MISALIGNED;
  uint32_t* status = status_ptr(&st);
  if (!status) return st;
  AttnParams prm{B, H, N, softmax_scale, sq, sk, sv, sv_max, out, out_dtype == FQA_OUT_F32, status};
  prm.q8 = static_cast<const uint8_t*>(q8);
  prm.k8 = static_cast<const uint8_t*>(k8);
  prm.kmask = nullptr;
  prm.row_stats = nullptr;
  return launch_attention_fp8(q8, k8, v8, prm, static_cast<cudaStream_t>(cuda_stream));
}

fqa_status fqa_attention_bf16(const void* q, const void* k, const void* v, int B, int H, int N,
                              int d, float softmax_scale, void* out, fqa_out_dtype out_dtype,
                              void* cuda_stream) {
  fqa_status st = check_attention_common(B, H, N, d, softmax_scale, out, out_dtype);
  if (st != FQA_OK) return st;
  const void* ptrs[] = {q, k, v};
  for (const void* p : ptrs) {
    if (p == nullptr) return FQA_ERR_INVALID_ARG;
    if (!aligned(p, 16)) return FQA_ERR_MISALIGNED;
  }
  uint32_t* status = status_ptr(&st);
  if (!status) return st;
  AttnParams prm{B, H, N, softmax_scale, nullptr, nullptr, nullptr, nullptr, out,
                 out_dtype == FQA_OUT_F32, status};
  return launch_attention_bf16(q, k, v, prm, static_cast<cudaStream_t>(cuda_stream));
}

// ------------------------------------------- sequence all-to-all layouts

// Shapes of the all-to-all calls: B, Hl heads, P chunks of Nl tokens
// (N = P * Nl), Nl a multiple of 64 so that no quantization block straddles
// two chunks.
static fqa_status check_a2a(int B, int Hl, int P, int Nl, int d) {
  if (P < 1 || Nl < 1) return FQA_ERR_INVALID_ARG;
  if (Nl % kQBlock != 0) return FQA_ERR_UNSUPPORTED;
  if ((int64_t)P * Nl > 65536) return FQA_ERR_UNSUPPORTED;
  return check_shape(B, Hl, P * Nl, d);
}

fqa_status fqa_quantize_a2a(const void* q, const void* k, const void* v, int B, int Hl, int P, int Nl, int d,
                            void* q8, void* k8, void* v8, float* sq, float* sk, float* sv, float* sv_max,
                            float* k_mean, void* workspace, size_t workspace_bytes, void* cuda_stream) {
  fqa_status st = check_a2a(B, Hl, P, Nl, d);
  if (st != FQA_OK) return st;
  return quantize_impl(q, k, v, B, Hl, P * Nl, d, q8, k8, v8, sq, sk, sv, sv_max, k_mean, nullptr, workspace,
                       workspace_bytes, cuda_stream, P);
}

fqa_status fqa_attention_fp8_a2a(const void* q8, const void* k8, const void* v8, const float* sq,
                                 const float* sk, const float* sv, const float* sv_max, int B, int Hl, int P,
                                 int Nl, int d, float softmax_scale, void* out, fqa_out_dtype out_dtype,
                                 void* cuda_stream) {
  fqa_status st = check_a2a(B, Hl, P, Nl, d);
  if (st != FQA_OK) return st;
  const int N = P * Nl;
  if ((st = check_attention_common(B, Hl, N, d, softmax_scale, out, out_dtype)) != FQA_OK) return st;
  const void* ptrs[] = {q8, k8, v8, sq, sk, sv, sv_max};
  for (const void* p : ptrs)
    if (p == nullptr) return FQA_ERR_INVALID_ARG;
  const void* a16[] = {q8, k8, v8};
  for (const void* p : a16)
    if (!aligned(p, 16)) return FQA_ERR_MISALIGNED;
  const void* a4[] = {sq, sk, sv, sv_max};
  for (const void* p : a4)
    if (!aligned(p, 4)) return FQA_ERR_MISALIGNED;
  uint32_t* status = status_ptr(&st);
  if (!status) return st;
  AttnParams prm{B, Hl, N, softmax_scale, sq, sk, sv, sv_max, out, out_dtype == FQA_OUT_F32, status};
  prm.q8 = static_cast<const uint8_t*>(q8);
  prm.k8 = static_cast<const uint8_t*>(k8);
  prm.out_P = P;
  return launch_attention_fp8(q8, k8, v8, prm, static_cast<cudaStream_t>(cuda_stream));
}

// ---------------------------------------------------- error-corrected path

// ceil(rho * N - 0.01): rho arrives in binary32, whose rounding moves rho * N
// by at most 0.004 for N <= 65536, so a product meant to be an integer (0.05
// of 1280 keys) stays that integer instead of rounding up.
int fqa_corrected_keys(int N, float rho) {
  if (N < 1 || !(rho >= 0.0f) || !(rho <= 1.0f)) return -1;
  const double kc = std::ceil((double)rho * (double)N - 0.01);
  return kc < 0.0 ? 0 : (kc > (double)N ? N : (int)kc);
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

fqa_status fqa_select_keys(const float* k_err, int B, int H, int N, int kc, uint32_t* kmask, int* idx,
                           void* cuda_stream) {
  fqa_status st = check_shape(B, H, N, 128);
  if (st != FQA_OK) return st;
  if (k_err == nullptr || kmask == nullptr || kc < 1 || kc > N || (idx == nullptr)) return FQA_ERR_INVALID_ARG;
  const void* a4[] = {k_err, kmask, idx};
  for (const void* p : a4)
    if (!aligned(p, 4)) return FQA_ERR_MISALIGNED;
  if (!status_ptr(&st)) return st;
  const int staged = N <= kSelStageMax ? 1 : 0;
  const int smem = staged ? N * 4 : 0;
  if (staged && cudaFuncSetAttribute(select_keys_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kSelStageMax * 4) != cudaSuccess)
    return FQA_ERR_CUDA;
  select_keys_kernel<<<B * H, kSelThreads, smem, static_cast<cudaStream_t>(cuda_stream)>>>(k_err, N, kc, kmask,
                                                                                         idx, staged);
  return launch_status();
}

size_t fqa_attention_fp8_corrected_workspace_bytes(int B, int H, int N, int d, float rho) {
  if (check_shape(B, H, N, d) != FQA_OK) return 0;
  const int kc = fqa_corrected_keys(N, rho);
  if (kc < 0) return 0;
  const size_t rows = (size_t)B * H * N;
  return align256((size_t)B * H * ((N + 31) / 32) * 4)      // key mask
         + align256((size_t)B * H * (size_t)(kc > 0 ? kc : 1) * 4)   // corrected indices
         + align256(rows * 8)                                // (m, l) per row
         + align256(rows * 128 * 4);                         // FP8 part, FP32
}

fqa_status fqa_attention_fp8_corrected(const void* q, const void* k, const void* v, const void* q8,
                                       const void* k8, const void* v8, const float* sq, const float* sk,
                                       const float* sv, const float* sv_max, const float* k_mean,
                                       const float* k_err, int B, int H, int N, int d, float softmax_scale,
                                       float rho, void* out, fqa_out_dtype out_dtype, void* workspace,
                                       size_t workspace_bytes, void* cuda_stream) {
  fqa_status st = check_attention_common(B, H, N, d, softmax_scale, out, out_dtype);
  if (st != FQA_OK) return st;
  const int kc = fqa_corrected_keys(N, rho);
  if (kc < 0) return FQA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, q8, k8, v8, sq, sk, sv, sv_max, k_mean, k_err, workspace};
  for (const void* p : ptrs)
    if (p == nullptr) return FQA_ERR_INVALID_ARG;
  if (workspace_bytes < fqa_attention_fp8_corrected_workspace_bytes(B, H, N, d, rho))
    return FQA_ERR_INVALID_ARG;
  const void* a16[] = {q, k, v, q8, k8, v8, workspace};
  for (const void* p : a16)
    if (!aligned(p, 16)) return FQA_ERR_MISALIGNED;
  const void* a4[] = {sq, sk, sv, sv_max, k_mean, k_err};
  for (const void* p : a4)
    if (!aligned(p, 4)) return FQA_ERR_MISALIGNED;
  uint32_t* status = status_ptr(&st);
  if (!status) return st;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  if (kc == 0)   // nothing to correct: the plain FP8 path
    return fqa_attention_fp8(q8, k8, v8, sq, sk, sv, sv_max, B, H, N, d, softmax_scale, out, out_dtype,
                             cuda_stream);
  // workspace: key mask | corrected indices | (m, l) | FP8 part (FP32)
  uint8_t* w = static_cast<uint8_t*>(workspace);
  uint32_t* kmask = reinterpret_cast<uint32_t*>(w);
  w += align256((size_t)B * H * ((N + 31) / 32) * 4);
  int* idx = reinterpret_cast<int*>(w);
  w += align256((size_t)B * H * (size_t)kc * 4);
  float2* stats = reinterpret_cast<float2*>(w);
  w += align256((size_t)B * H * N * 8);
  float* o1 = reinterpret_cast<float*>(w);
  if ((st = fqa_select_keys(k_err, B, H, N, kc, kmask, idx, cuda_stream)) != FQA_OK) return st;
  AttnParams prm{B, H, N, softmax_scale, sq, sk, sv, sv_max, o1, 1, status};
  prm.q8 = static_cast<const uint8_t*>(q8);
  prm.k8 = static_cast<const uint8_t*>(k8);
  prm.kmask = kmask;
  prm.row_stats = stats;
  // fewer than 64 corrected keys per head leave a kept key in every 64-key
  // block: the key mask can be applied by patching tiles
  prm.patch = (kc < 64 && N % kBlockN == 0) ? 1 : 0;
  if ((st = launch_attention_fp8(q8, k8, v8, prm, s)) != FQA_OK) return st;
  if (prm.patch) {
    // take the copied keys' terms out of the patched FP8 part's row sums
    CUtensorMap tq8;
    if (!make_tmap(&tq8, q8, true, N, B * H)) return FQA_ERR_CUDA;
    if (cudaFuncSetAttribute(dup_sum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDupSmem) !=
        cudaSuccess)
      return FQA_ERR_CUDA;
    DupParams dp{static_cast<const uint8_t*>(k8), sq, sk, kmask, stats, N, softmax_scale, status};
    dup_sum_kernel<<<dim3(N / kBlockM, B * H), kDupThreads, kDupSmem, s>>>(tq8, dp);
    if ((st = launch_status()) != FQA_OK) return st;
  }
  // exact part over the corrected keys, merged into the output: one chunk of
  // 64 (two CTAs per SM; three of its rows carry the K mean) when they fit
  CUtensorMap tq;
  if (!make_tmap(&tq, q, false, N, B * H)) return FQA_ERR_CUDA;
  CorrParams cp{static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                static_cast<const __nv_bfloat16*>(v), k_mean, idx, o1, stats, prm.patch, out,
                out_dtype == FQA_OUT_F32, B, H, N, kc, softmax_scale, status};
  const bool small = kc <= 61;
  const void* fn = small ? (const void*)correct_kernel<64> : (const void*)correct_kernel<128>;
  const int smem = small ? CorrTraits<64>::kSmemBytes : CorrTraits<128>::kSmemBytes;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return FQA_ERR_CUDA;
  const int sms = num_sms() * (small ? CorrTraits<64>::kCtasPerSm : CorrTraits<128>::kCtasPerSm);
  const int ntq = (N + 127) / 128;
  int split = (sms + B * H - 1) / (B * H);       // about one wave of CTAs
  if (split > ntq) split = ntq;
  if (split < 1) split = 1;
  if (small)
    correct_kernel<64><<<dim3(split, B * H), kCorrThreads, smem, s>>>(tq, cp);
  else
    correct_kernel<128><<<dim3(split, B * H), kCorrThreads, smem, s>>>(tq, cp);
  return launch_status();
}

// ------------------------------------------------------- NVFP4 Q.K variant

fqa_status fqa_quantize_nvfp4_qk(const void* q, const void* k, const float* k_mean, int B, int H, int N, int d,
                                 uint8_t* q4, uint8_t* k4, uint8_t* sfq, uint8_t* sfk, float* sq1, float* sk1,
                                 void* cuda_stream) {
  fqa_status st = check_shape(B, H, N, d);
  if (st != FQA_OK) return st;
  const void* ptrs[] = {q, k, k_mean, q4, k4, sfq, sfk, sq1, sk1};
  for (const void* p : ptrs)
    if (p == nullptr) return FQA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16)) return FQA_ERR_MISALIGNED;
  const void* a4[] = {k_mean, q4, k4, sq1, sk1};
  for (const void* p : a4)
    if (!aligned(p, 4)) return FQA_ERR_MISALIGNED;
  const int units = B * H * ((N + 63) / 64);
  quantize_nvfp4_kernel<<<2 * units, kNv4Threads, 0, static_cast<cudaStream_t>(cuda_stream)>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), k_mean, q4, k4, sfq, sfk,
      sq1, sk1, B, H, N);
  return launch_status();
}

fqa_status fqa_attention_nvfp4(const uint8_t* q4, const uint8_t* k4, const uint8_t* sfq, const uint8_t* sfk,
                               const float* sq1, const float* sk1, const void* v8, const float* sv,
                               const float* sv_max, int B, int H, int N, int d, float softmax_scale, void* out,
                               fqa_out_dtype out_dtype, void* cuda_stream) {
  fqa_status st = check_attention_common(B, H, N, d, softmax_scale, out, out_dtype);
  if (st != FQA_OK) return st;
  const void* ptrs[] = {q4, k4, sfq, sfk, sq1, sk1, v8, sv, sv_max};
  for (const void* p : ptrs)
    if (p == nullptr) return FQA_ERR_INVALID_ARG;
  const void* a16[] = {q4, k4, v8};
  for (const void* p : a16)
    if (!aligned(p, 16)) return FQA_ERR_MISALIGNED;
  if (!aligned(sfq, 8) || !aligned(sfk, 8)) return FQA_ERR_MISALIGNED;
  const void* a4[] = {sq1, sk1, sv, sv_max};
  for (const void* p : a4)
    if (!aligned(p, 4)) return FQA_ERR_MISALIGNED;
  uint32_t* status = status_ptr(&st);
  if (!status) return st;
  const int heads = B * H;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_fp4(&tq, q4, N, heads) || !make_tmap_fp4(&tk, k4, N, heads) ||
      !make_tmap(&tv, v8, true, N, heads))
    return FQA_ERR_CUDA;
  // the short-tail instance only when N is not a multiple of 128
  const bool tail = N % kBlockN != 0;
  using NvKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const NvParams);
  const NvKernel fn = tail ? attn_nvfp4_kernel<true> : attn_nvfp4_kernel<false>;
  if (cudaFuncSetAttribute((const void*)fn, cudaFuncAttributeMaxDynamicSharedMemorySize, NvTraits::kSmemBytes) !=
      cudaSuccess)
    return FQA_ERR_CUDA;
  NvParams prm{B, H, N, softmax_scale, sfq, sfk, sq1, sk1, sv, sv_max, out, out_dtype == FQA_OUT_F32, status};
  const int items = heads * ((N + kBlockM - 1) / kBlockM);
  const int sms = num_sms();
  if (sms <= 0) return FQA_ERR_CUDA;
  const int grid = items < sms ? items : sms;
  fn<<<grid, kNvThreads, NvTraits::kSmemBytes, static_cast<cudaStream_t>(cuda_stream)>>>(tq, tk, tv, prm);
  return launch_status();
}

fqa_status fqa_e2m1_encode(const float* x, uint8_t* out, size_t npairs, void* cuda_stream) {
  if (x == nullptr || out == nullptr) return FQA_ERR_INVALID_ARG;
  if (npairs == 0) return FQA_OK;
  if (!aligned(x, 8)) return FQA_ERR_MISALIGNED;
  e2m1_encode_kernel<<<148 * 8, 256, 0, static_cast<cudaStream_t>(cuda_stream)>>>(x, out, npairs);
  return launch_status();
}

fqa_status fqa_exp2_error(float lo, float hi, uint32_t* max_rel_bits, void* cuda_stream) {
  if (max_rel_bits == nullptr) return FQA_ERR_INVALID_ARG;
  if (!(lo <= hi) || !(hi <= 0.0f) || !(lo >= -126.0f)) return FQA_ERR_INVALID_ARG;
  if (!aligned(max_rel_bits, 4)) return FQA_ERR_MISALIGNED;
  // negative binary32 values from hi down to lo are consecutive bit patterns
  uint32_t hb, lb;
  const float h = hi == 0.0f ? -0.0f : hi;
  std::memcpy(&hb, &h, 4);
  std::memcpy(&lb, &lo, 4);
  const uint32_t n = lb - hb + 1;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  if (cudaMemsetAsync(max_rel_bits, 0, 4, s) != cudaSuccess) return FQA_ERR_CUDA;
  exp2_error_kernel<<<148 * 16, 256, 0, s>>>(lb, n, reinterpret_cast<unsigned int*>(max_rel_bits));
  return launch_status();
}

fqa_status fqa_e4m3_encode(const float* x, uint8_t* out, size_t n, void* cuda_stream) {
  if (x == nullptr || out == nullptr) return FQA_ERR_INVALID_ARG;
  if (n == 0) return FQA_OK;
  if (!aligned(x, 4)) return FQA_ERR_MISALIGNED;
  e4m3_encode_kernel<<<148 * 8, 256, 0, static_cast<cudaStream_t>(cuda_stream)>>>(x, out, n);
  return launch_status();
}

fqa_status fqa_debug_wait_timeout(uint32_t limit_us, void* cuda_stream) {
  if (limit_us == 0 || limit_us > 2000000u) return FQA_ERR_INVALID_ARG;
  fqa_status st = FQA_OK;
  uint32_t* status = status_ptr(&st);
  if (!status) return st;
  wait_timeout_kernel<<<1, 1, 0, static_cast<cudaStream_t>(cuda_stream)>>>(
      status, (uint64_t)limit_us * 1000ull);
  return launch_status();
}

fqa_status fqa_debug_status(void* cuda_stream, uint32_t* flags_out) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return FQA_ERR_CUDA;
  uint32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof(v)) != cudaSuccess) return FQA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero)) != cudaSuccess) return FQA_ERR_CUDA;
  if (flags_out) *flags_out = v;
  return (v & kStatusTimeout) ? FQA_ERR_TIMEOUT : FQA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// fqa_quantize_noalloc: fqa_quantize for callers that cannot allocate device
// memory when they call.  The K-mean partial sums live in a fixed array inside
// the library instead of a caller-provided workspace.
namespace fqa {

// The scratch fqa_quantize needs is the K-mean partial sums,
// B*H*ceil(N/64)*128*4 bytes rounded up to 256, plus 256 bytes of counters.
// 8 MiB of partial sums covers B*H*ceil(N/64) <= 16384 blocks (B=2, H=24,
// N=16896 needs 6.2 MiB); the array holds that plus the counters.
constexpr size_t kNoAllocScratchBytes = (size_t(8) << 20) + 256;

// One copy per GPU that loads the library, held until the process exits.
// In host code this name is only a stand-in: the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

struct NoAllocCache {
  std::mutex mu;
  float* ptr = nullptr;
};
NoAllocCache g_noalloc[kMaxDevices];

// Device address of this device's scratch array, looked up with that device
// current; cached once the lookup succeeds (a failed lookup, e.g. during a
// stream capture, is retried by the next call).
static float* noalloc_scratch(fqa_status* st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *st = FQA_ERR_CUDA;
    return nullptr;
  }
  NoAllocCache& c = g_noalloc[dev];
  std::lock_guard<std::mutex> lock(c.mu);
  if (c.ptr == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      *st = FQA_ERR_CUDA;
      return nullptr;
    }
    c.ptr = static_cast<float*>(p);
  }
  return c.ptr;
}

}  // namespace fqa

extern "C" size_t fqa_quantize_noalloc_max_workspace_bytes(void) { return kNoAllocScratchBytes; }

extern "C" fqa_status fqa_quantize_noalloc(const void* q, const void* k, const void* v, int B, int H,
                                           int N, int d, void* q8, void* k8, void* v8, float* sq,
                                           float* sk, float* sv, float* sv_max, float* k_mean,
                                           void* cuda_stream) {
  fqa_status st = check_shape(B, H, N, d);
  if (st != FQA_OK) return st;
  if (fqa_quantize_workspace_bytes(B, H, N, d) > kNoAllocScratchBytes) return FQA_ERR_UNSUPPORTED;
  float* scratch = noalloc_scratch(&st);
  if (scratch == nullptr) return st;
  return fqa_quantize(q, k, v, B, H, N, d, q8, k8, v8, sq, sk, sv, sv_max, k_mean, scratch,
                      kNoAllocScratchBytes, cuda_stream);
}
