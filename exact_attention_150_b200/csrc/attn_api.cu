// attn_api.cu -- the C ABI declared in include/attn.h: host-side argument
// validation, TMA tensor-map construction and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "bwd_kernel.cuh"
#include "fwd_kernel.cuh"

namespace {

using attn::kTile;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3D view [B*H][N][d] of a contiguous 16-bit tensor, read in boxes of 64
// columns (128 bytes) x 128 rows of one (b, h) slice with the 128-byte
// swizzle the MMA descriptors expect.  Rows past N read as zeros, so a
// ragged last tile never touches the next slice.
bool make_map(CUtensorMap* map, const void* base, int BH, int N, int d, bool bf16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kTile), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int tiles(int n) { return (n + kTile - 1) / kTile; }

// Rows after the dQ accumulator that a ragged last query tile of the last
// (b, h) slice reduces into.  The main kernel reduces all 128 rows of every
// query tile without a per-row test; the rows past Nq carry exact zeros
// (their probabilities are masked and their dO rows read as zeros), so in
// other slices they land harmlessly on the next slice's first rows, and in
// the last slice they land here.
long long pad_rows(int Nq) { return static_cast<long long>(tiles(Nq)) * kTile - Nq; }

// Workspace layout: dQ accumulator [(B*H*Nq + pad_rows) * d] | D [B*H*Nq] |
// -log2(e) LSE [B*H*Nq] | (16-byte aligned) order counters [B*H][tiles(Nq)]
// of the deterministic backward.
long long counters_offset_floats(int BH, int Nq, int d) {
  const long long rows = static_cast<long long>(BH) * Nq;
  const long long f = (rows + pad_rows(Nq)) * d + 2 * rows;
  return (f + 3) / 4 * 4;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Sizes may be zero (an empty problem); they may not be negative.
attn_status check_common(int B, int H, int Nq, int Nk, int d, int causal, attn_dtype dtype) {
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || d < 0) return ATTN_ERR_INVALID_ARG;
  if (causal != ATTN_CAUSAL_NONE && causal != ATTN_CAUSAL_TOP_LEFT && causal != ATTN_CAUSAL_BOTTOM_RIGHT)
    return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_FP16 && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  const long long bh = static_cast<long long>(B) * H;
  // Grid x and TMA coordinates are 32-bit; grid y is 16-bit.
  if (bh > 0x7fffffffLL || tiles(Nq) > 65535 || tiles(Nk) > 65535) return ATTN_ERR_UNSUPPORTED;
  if (bh * Nq > (1LL << 40) || bh * Nk > (1LL << 40)) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int D, bool BF16, bool CAUSAL>
attn_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, void* o, float* lse,
                       int BH, int Nq, int Nk, int off, float scale_log2, cudaStream_t st) {
  using L = attn::FwdLayout<D>;
  auto kern = attn::fwd_kernel<D, BF16, CAUSAL>;
  if (set_smem(kern, L::kAlloc) != cudaSuccess) return ATTN_ERR_CUDA;
  dim3 grid(BH, tiles(Nq));
  kern<<<grid, 384, L::kAlloc, st>>>(mq, mk, mv, static_cast<uint16_t*>(o), lse, Nq, Nk, off, scale_log2);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool BF16, bool CAUSAL, bool DET>
attn_status launch_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                       const void* o, const void* dout, const float* lse, void* dq, void* dk, void* dv, float* ws,
                       int BH, int Nq, int Nk, int off, float scale, int phase, cudaStream_t st) {
  using L = attn::BwdLayout<D>;
  const long long qrows = static_cast<long long>(BH) * Nq;
  float* dqacc = ws;
  float* dvec = ws + (qrows + pad_rows(Nq)) * D;
  float* nlse2 = dvec + qrows;
  int* dq_order = DET ? reinterpret_cast<int*>(ws + counters_offset_floats(BH, Nq, D)) : nullptr;

  if (phase == ATTN_BWD_ALL || phase == ATTN_BWD_PREPROCESS) {
    if (DET && cudaMemsetAsync(dq_order, 0, static_cast<size_t>(BH) * tiles(Nq) * sizeof(int), st) != cudaSuccess)
      return ATTN_ERR_CUDA;
    constexpr int kRowsPerBlock = 256 / (D / 8);
    const long long pre_blocks = (qrows + kRowsPerBlock - 1) / kRowsPerBlock;
    attn::bwd_pre_kernel<D, BF16><<<static_cast<unsigned>(pre_blocks), 256, 0, st>>>(
        static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse, dvec, nlse2, dqacc, qrows);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (phase == ATTN_BWD_ALL || phase == ATTN_BWD_MAIN) {
    auto kern = attn::bwd_main_kernel<D, BF16, CAUSAL, DET>;
    if (set_smem(kern, L::kAlloc) != cudaSuccess) return ATTN_ERR_CUDA;
    dim3 grid(BH, tiles(Nk));
    kern<<<grid, 512, L::kAlloc, st>>>(mq, mk, mv, mdo, dvec, nlse2, dqacc, static_cast<uint16_t*>(dk),
                                       static_cast<uint16_t*>(dv), dq_order, Nq, Nk, off, scale,
                                       scale * 1.4426950408889634f);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (phase == ATTN_BWD_ALL || phase == ATTN_BWD_CONVERT) {
    const long long n8 = qrows * D / 8;
    long long post_blocks = (n8 + 255) / 256;
    if (post_blocks > 148LL * 16) post_blocks = 148LL * 16;
    attn::bwd_post_kernel<BF16>
        <<<static_cast<unsigned>(post_blocks), 256, 0, st>>>(dqacc, static_cast<uint16_t*>(dq), n8);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

// Diagonal offset of the causal mask: query i sees key k iff k <= i + off.
int causal_offset(int causal, int Nq, int Nk) { return causal == ATTN_CAUSAL_BOTTOM_RIGHT ? Nk - Nq : 0; }

template <int D, bool BF16>
attn_status dispatch_fwd_causal(int causal, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                void* o, float* lse, int BH, int Nq, int Nk, float sl2, cudaStream_t st) {
  const int off = causal_offset(causal, Nq, Nk);
  return causal ? launch_fwd<D, BF16, true>(mq, mk, mv, o, lse, BH, Nq, Nk, off, sl2, st)
                : launch_fwd<D, BF16, false>(mq, mk, mv, o, lse, BH, Nq, Nk, off, sl2, st);
}

template <int D, bool BF16>
attn_status dispatch_bwd_causal(int causal, bool det, const CUtensorMap& mq, const CUtensorMap& mk,
                                const CUtensorMap& mv, const CUtensorMap& mdo, const void* o, const void* dout,
                                const float* lse, void* dq, void* dk, void* dv, float* ws, int BH, int Nq, int Nk,
                                float scale, int phase, cudaStream_t st) {
  const int off = causal_offset(causal, Nq, Nk);
#define ATTN_LAUNCH_BWD(C, DT) \
  launch_bwd<D, BF16, C, DT>(mq, mk, mv, mdo, o, dout, lse, dq, dk, dv, ws, BH, Nq, Nk, off, scale, phase, st)
  if (det) return causal ? ATTN_LAUNCH_BWD(true, true) : ATTN_LAUNCH_BWD(false, true);
  return causal ? ATTN_LAUNCH_BWD(true, false) : ATTN_LAUNCH_BWD(false, false);
#undef ATTN_LAUNCH_BWD
}

// The backward phases shared by attn_bwd_phase (det = false) and
// attn_bwd_deterministic (det = true).
attn_status bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, void* workspace, int B, int H, int Nq, int Nk, int d, float scale,
                     int causal, attn_dtype dtype, int phase, bool det, void* stream);

}  // namespace

// ------------------------------------------------ allocation-free backward
//
// attn_bwd_noalloc runs the backward pass with its workspace in this fixed
// array instead of a caller-provided buffer.  It exists for callers that
// cannot allocate device memory when they call: a plugin inside another
// runtime's execution callback that must not allocate, or a process whose
// device memory is entirely held by another allocator's pool.  The array is
// part of this library's module, so every GPU that loads the library holds
// it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(72) << 20;  // 72 MiB
static __device__ __align__(256) unsigned char g_bwd_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// In host code g_bwd_scratch is only a host-side stand-in for the device
// array: its device address is looked up once per device, with that device
// current, and cached.
attn_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) return ATTN_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" {

attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                     int d, float scale, int causal, attn_dtype dtype, void* stream) {
  const attn_status cs = check_common(B, H, Nq, Nk, d, causal, dtype);
  if (cs != ATTN_OK) return cs;
  if (B == 0 || H == 0 || Nq == 0) return ATTN_OK;  // no query rows: nothing to write
  if (Nk == 0) return ATTN_ERR_INVALID_ARG;         // a softmax over no keys is undefined
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_INVALID_ARG;
  const bool bf16 = dtype == ATTN_BF16;
  const int BH = B * H;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, BH, Nq, d, bf16) || !make_map(&mk, k, BH, Nk, d, bf16) || !make_map(&mv, v, BH, Nk, d, bf16))
    return ATTN_ERR_CUDA;
  const float sl2 = scale * 1.4426950408889634f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 64)
    return bf16 ? dispatch_fwd_causal<64, true>(causal, mq, mk, mv, o, lse, BH, Nq, Nk, sl2, st)
                : dispatch_fwd_causal<64, false>(causal, mq, mk, mv, o, lse, BH, Nq, Nk, sl2, st);
  return bf16 ? dispatch_fwd_causal<128, true>(causal, mq, mk, mv, o, lse, BH, Nq, Nk, sl2, st)
              : dispatch_fwd_causal<128, false>(causal, mq, mk, mv, o, lse, BH, Nq, Nk, sl2, st);
}

size_t attn_bwd_workspace_bytes(int B, int H, int Nq, int Nk, int d) {
  if (B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return 0;  // empty problems need none
  const long long bh = static_cast<long long>(B) * H;
  if (bh > 0x7fffffffLL || bh * Nq > (1LL << 40)) return 0;
  const unsigned long long words = static_cast<unsigned long long>(counters_offset_floats(static_cast<int>(bh), Nq, d)) +
                                   static_cast<unsigned long long>(bh) * tiles(Nq);
  return static_cast<size_t>(words * 4);
}

attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, void* workspace, int B, int H, int Nq, int Nk, int d, float scale,
                     int causal, attn_dtype dtype, void* stream) {
  return attn_bwd_phase(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, Nq, Nk, d, scale, causal, dtype,
                        ATTN_BWD_ALL, stream);
}

attn_status attn_bwd_phase(const void* q, const void* k, const void* v, const void* o, const float* lse,
                           const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int H, int Nq,
                           int Nk, int d, float scale, int causal, attn_dtype dtype, int phase, void* stream) {
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, Nq, Nk, d, scale, causal, dtype, phase, false,
                  stream);
}

attn_status attn_bwd_deterministic(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                   const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int H,
                                   int Nq, int Nk, int d, float scale, int causal, attn_dtype dtype, void* stream) {
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, Nq, Nk, d, scale, causal, dtype, ATTN_BWD_ALL,
                  true, stream);
}

}  // extern "C"

namespace {

attn_status bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, void* workspace, int B, int H, int Nq, int Nk, int d, float scale,
                     int causal, attn_dtype dtype, int phase, bool det, void* stream) {
  if (phase < ATTN_BWD_ALL || phase > ATTN_BWD_CONVERT) return ATTN_ERR_INVALID_ARG;
  const attn_status cs = check_common(B, H, Nq, Nk, d, causal, dtype);
  if (cs != ATTN_OK) return cs;
  if (B == 0 || H == 0) return ATTN_OK;
  if (Nk == 0) return Nq == 0 ? ATTN_OK : ATTN_ERR_INVALID_ARG;
  cudaStream_t st0 = static_cast<cudaStream_t>(stream);
  if (Nq == 0) {
    // No query rows: dK = dV = 0 (written by the main phase), dQ is empty.
    if (!dk || !dv) return ATTN_ERR_INVALID_ARG;
    if (phase != ATTN_BWD_ALL && phase != ATTN_BWD_MAIN) return ATTN_OK;
    const size_t bytes = static_cast<size_t>(B) * H * Nk * d * 2;
    if (cudaMemsetAsync(dk, 0, bytes, st0) != cudaSuccess || cudaMemsetAsync(dv, 0, bytes, st0) != cudaSuccess)
      return ATTN_ERR_CUDA;
    return ATTN_OK;
  }
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace) return ATTN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return ATTN_ERR_INVALID_ARG;
  const bool bf16 = dtype == ATTN_BF16;
  const int BH = B * H;
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, q, BH, Nq, d, bf16) || !make_map(&mk, k, BH, Nk, d, bf16) ||
      !make_map(&mv, v, BH, Nk, d, bf16) || !make_map(&mdo, dout, BH, Nq, d, bf16))
    return ATTN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
#define ATTN_DISPATCH_BWD(DD, BB) \
  dispatch_bwd_causal<DD, BB>(causal, det, mq, mk, mv, mdo, o, dout, lse, dq, dk, dv, ws, BH, Nq, Nk, scale, phase, st)
  if (d == 64) return bf16 ? ATTN_DISPATCH_BWD(64, true) : ATTN_DISPATCH_BWD(64, false);
  return bf16 ? ATTN_DISPATCH_BWD(128, true) : ATTN_DISPATCH_BWD(128, false);
#undef ATTN_DISPATCH_BWD
}

}  // namespace

extern "C" {

attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                             const void* dout, void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int d,
                             float scale, int causal, attn_dtype dtype, void* stream) {
  const attn_status cs = check_common(B, H, Nq, Nk, d, causal, dtype);
  if (cs != ATTN_OK) return cs;
  if (attn_bwd_workspace_bytes(B, H, Nq, Nk, d) > kNoAllocScratchBytes) return ATTN_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if (B > 0 && H > 0 && Nq > 0 && Nk > 0) {
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
    const attn_status ss = scratch_for_current_device(&scratch);
    if (ss != ATTN_OK) return ss;
  }
  // The preprocess kernel rewrites every byte of the scratch that the main
  // kernel reads (it zeroes the dQ accumulator), so the previous call's
  // contents never leak into this one.
  return attn_bwd_phase(q, k, v, o, lse, dout, dq, dk, dv, scratch, B, H, Nq, Nk, d, scale, causal, dtype,
                        ATTN_BWD_ALL, stream);
}

size_t attn_bwd_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

attn_status attn_last_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  int status = 0;
  if (cudaMemcpyFromSymbol(&status, attn::g_device_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (status != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(attn::g_device_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return static_cast<attn_status>(status);
}

const char* attn_status_string(attn_status s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_TIMEOUT: return "device wait timed out";
    case ATTN_ERR_SMEM: return "kernel found less shared memory than its tiles need";
    case ATTN_ERR_SCRATCH_LIMIT: return "problem needs more scratch than attn_bwd_noalloc's fixed 72 MiB array";
  }
  return "unknown status";
}

}  // extern "C"
