// attn_api.cu -- the C ABI declared in include/attn.h: host-side argument
// validation, TMA tensor-map construction and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include "attn.h"
#include "bwd_dq_kernel.cuh"
#include "bwd_kernel.cuh"
#include "bwd_kv_wide_kernel.cuh"
#include "fwd_kernel.cuh"
#include "trace.h"

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

// 3D view [slabs][N][d] of a contiguous 16-bit (or, with e4m3, 8-bit)
// tensor (a slab is one (batch, head) slice of a dense batch, or one head of
// a packed variable-length batch), read in boxes 128 bytes wide (64 16-bit
// or 128 8-bit columns) x box_rows rows of one slab, with the 128-byte
// swizzle the MMA descriptors expect.  Rows past N read as zeros, so a
// ragged last tile never touches the next slab.
bool make_map(CUtensorMap* map, const void* base, int BH, int N, int d, bool bf16, bool e4m3 = false,
              int box_rows = kTile) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t eb = e4m3 ? 1 : 2;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * eb, static_cast<cuuint64_t>(N) * d * eb};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / eb), static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType type = e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                        : (bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  const CUresult r = fn(map, type, 3,
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


bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Sizes may be zero (an empty problem); they may not be negative.
attn_status check_common(int B, int H, int Nq, int Nk, int d, int causal, attn_dtype dtype) {
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || d < 0) return ATTN_ERR_INVALID_ARG;
  if (causal != ATTN_CAUSAL_NONE && causal != ATTN_CAUSAL_TOP_LEFT && causal != ATTN_CAUSAL_BOTTOM_RIGHT)
    return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_FP16 && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  const long long bh = static_cast<long long>(B) * H;
  // TMA coordinates are 32-bit, and so is the one-dimensional grid of
  // (problem, tile) CTAs.
  if (bh > 0x7fffffffLL || tiles(Nq) > 65535 || tiles(Nk) > 65535) return ATTN_ERR_UNSUPPORTED;
  if (bh * tiles(Nq) > 0x7fffffffLL || bh * tiles(Nk) > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (bh * Nq > (1LL << 40) || bh * Nk > (1LL << 40)) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

// Multiprocessor count of the current device (0 if it cannot be read),
// read once per device.
int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64 && (n = cached[dev].load(std::memory_order_relaxed)) > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Raises a kernel's dynamic shared-memory limit once per (kernel, device):
// the attribute persists, and setting it on every launch costs host time
// that small problems notice.

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  const cudaError_t ge = cudaGetDevice(&dev);
  if (ge != cudaSuccess) return ge;
  const std::pair<const void*, int> key(reinterpret_cast<const void*>(kernel), dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    if (done.count(key)) return cudaSuccess;
  }
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) {
    std::lock_guard<std::mutex> lock(mu);
    done.insert(key);
  }
  return e;
}

// A launch's problems.  Dense batches: one tensor-map slab per (batch,
// head), all of its rows.  Packed variable-length batches: one slab per
// head; problem b*H + h is sequence b of head h, whose rows the kernels take
// from the device offsets cu_q / cu_k.
struct Problem {
  int slabs;               // slab count of the tensor maps
  int rows_q, rows_k;      // rows per slab
  int problems;            // B*H
  int qtiles, ktiles;      // tiles of the longest query / key sequence
  const int* cu_q = nullptr;
  const int* cu_k = nullptr;
  int H = 1;
  int bottom_right = 0;
  bool packed = false;     // variable-length batch
};

// Average rows per problem of a tensor with rows_per_slab rows in each slab.
double avg_rows(int rows_per_slab, const Problem& pb) {
  return pb.problems > 0 ? static_cast<double>(rows_per_slab) * pb.slabs / pb.problems : 0.0;
}

Problem dense_problem(int B, int H, int Nq, int Nk, int causal) {
  Problem p;
  p.slabs = p.problems = B * H;
  p.rows_q = Nq;
  p.rows_k = Nk;
  p.qtiles = tiles(Nq);
  p.ktiles = tiles(Nk);
  p.bottom_right = causal == ATTN_CAUSAL_BOTTOM_RIGHT;
  return p;
}

// Packed variable-length batches: sizes may be zero, not negative; the
// offsets themselves live on the device and are clamped by the kernels.
attn_status check_varlen(int B, int H, int total_q, int total_k, int max_q, int max_k, int d, int causal,
                         attn_dtype dtype) {
  if (B < 0 || H < 0 || total_q < 0 || total_k < 0 || max_q < 0 || max_k < 0 || d < 0) return ATTN_ERR_INVALID_ARG;
  if (causal != ATTN_CAUSAL_NONE && causal != ATTN_CAUSAL_TOP_LEFT && causal != ATTN_CAUSAL_BOTTOM_RIGHT)
    return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_FP16 && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  const long long bh = static_cast<long long>(B) * H;
  if (bh > 0x7fffffffLL || tiles(max_q) > 65535 || tiles(max_k) > 65535) return ATTN_ERR_UNSUPPORTED;
  if (bh * tiles(max_q) > 0x7fffffffLL || bh * tiles(max_k) > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(H) * total_q > (1LL << 40) || static_cast<long long>(H) * total_k > (1LL << 40))
    return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

Problem varlen_problem(int B, int H, int total_q, int total_k, int max_q, int max_k, const int* cu_q,
                       const int* cu_k, int causal) {
  Problem p;
  p.slabs = H;
  p.rows_q = total_q;
  p.rows_k = total_k;
  p.problems = B * H;
  p.qtiles = tiles(max_q);
  p.ktiles = tiles(max_k);
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.H = H;
  p.bottom_right = causal == ATTN_CAUSAL_BOTTOM_RIGHT;
  p.packed = true;
  return p;
}

// Backward workspace of a problem, in 4-byte words: dQ accumulator
// [(rows + pad) * d] | D [rows] | -log2(e) LSE [rows] | (16-byte aligned)
// [problems][qtiles] words that no kernel uses at present (they keep the
// size attn_bwd_workspace_bytes documents), with rows = slabs * rows_q.
// The pad takes the reductions of the ragged last query tile's masked rows
// (exact zeros; see pad_rows); in a packed batch any sequence's last tile
// can reach up to 127 rows past the total.  The reproducible backward and
// every d = 256 backward leave the accumulator unused.
struct WsLayout {
  long long rows, dvec, nlse2, counters, ncounters, words;
};

WsLayout ws_layout(const Problem& pb, int d) {
  WsLayout w;
  w.rows = static_cast<long long>(pb.slabs) * pb.rows_q;
  const long long pad = pb.packed ? kTile : pad_rows(pb.rows_q);
  w.dvec = (w.rows + pad) * d;
  w.nlse2 = w.dvec + w.rows;
  w.counters = (w.nlse2 + w.rows + 3) / 4 * 4;
  w.ncounters = static_cast<long long>(pb.problems) * pb.qtiles;
  w.words = w.counters + w.ncounters;
  return w;
}

template <int D, bool BF16, bool CAUSAL, bool F8 = false>
attn_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                       void* o, float* lse, const Problem& pb, float scale_log2, cudaStream_t st,
                       float o_scale = 1.f) {
  using L = attn::FwdLayout<D, F8>;
  auto kern = attn::fwd_kernel<D, BF16, CAUSAL, F8>;
  if (set_smem(kern, L::kAlloc) != cudaSuccess) return ATTN_ERR_CUDA;
  // Every CTA of a problem streams its K and V.
  const int group = attn::order_group(2.0 * L::kRowBytes * avg_rows(pb.rows_k, pb), pb.problems);
  // Persistent: one CTA per SM (the shared memory and the 512 tensor-memory
  // columns allow no second), each walking its share of the query tiles.
  const unsigned units = static_cast<unsigned>(pb.problems) * static_cast<unsigned>(pb.qtiles);
  const unsigned sms = static_cast<unsigned>(sm_count());
  if (sms == 0) return ATTN_ERR_CUDA;
  const unsigned grid = units < sms ? units : sms;
  // Causal grids with at least two units per CTA deal heavy and light tiles
  // out in pairs (tile_order.h).
  const int fold = CAUSAL && units >= 2u * sms ? 1 : 0;
  kern<<<grid, 384, L::kAlloc, st>>>(mq, mk, mv, mo, static_cast<uint16_t*>(o), lse, pb.cu_q, pb.cu_k, pb.H, pb.rows_q,
                                     pb.rows_k, pb.bottom_right, scale_log2, pb.problems, pb.qtiles, group, fold,
                                     o_scale);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// The backward kernels of one call.  DET = false: preprocess (which also
// zeroes the fp32 dQ accumulator), the main kernel with atomic dQ
// reductions, and the dQ convert.  DET = true: preprocess, the main kernel
// for dK and dV only, and the dQ kernel, which owns its dQ rows and writes
// them directly (no accumulator, no atomics, the same bits on every run).
template <int D, bool BF16, bool CAUSAL, bool DET>
attn_status launch_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                       const void* o, const void* dout, const float* lse, void* dq, void* dk, void* dv, float* ws,
                       const Problem& pb, float scale, int phase, cudaStream_t st) {
  using L = attn::BwdLayout<D>;
  const WsLayout w = ws_layout(pb, D);
  const long long qrows = w.rows;
  float* dqacc = ws;
  float* dvec = ws + w.dvec;
  float* nlse2 = ws + w.nlse2;
  const float scale_log2 = scale * 1.4426950408889634f;

  if (phase == ATTN_BWD_ALL || phase == ATTN_BWD_PREPROCESS) {
    constexpr int kRowsPerBlock = 256 / (D / 8);
    const long long pre_blocks = (qrows + kRowsPerBlock - 1) / kRowsPerBlock;
    attn::bwd_pre_kernel<D, BF16><<<static_cast<unsigned>(pre_blocks), 256, 0, st>>>(
        static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse, dvec, nlse2, DET ? nullptr : dqacc,
        qrows);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (phase == ATTN_BWD_ALL || phase == ATTN_BWD_MAIN) {
    auto kern = attn::bwd_main_kernel<D, BF16, CAUSAL, !DET>;
    if (set_smem(kern, L::kAlloc) != cudaSuccess) return ATTN_ERR_CUDA;
    // Every CTA of a problem streams its Q and dO rows, their LSE and D, and
    // (atomic dQ) adds into its dQ accumulator rows.
    const int group = attn::order_group((8.0 * D + 8.0) * avg_rows(pb.rows_q, pb), pb.problems);
    const unsigned grid = static_cast<unsigned>(pb.problems) * static_cast<unsigned>(pb.ktiles);
    kern<<<grid, 512, L::kAlloc, st>>>(mq, mk, mv, mdo, dvec, nlse2, dqacc, static_cast<uint16_t*>(dk),
                                       static_cast<uint16_t*>(dv), pb.cu_q, pb.cu_k, pb.H, pb.rows_q, pb.rows_k,
                                       pb.bottom_right, pb.qtiles, scale, scale_log2, pb.problems, pb.ktiles, group);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    if constexpr (DET) {
      using LQ = attn::BwdDqLayout<D>;
      auto kq = attn::bwd_dq_kernel<D, BF16, CAUSAL>;
      if (set_smem(kq, LQ::kAlloc) != cudaSuccess) return ATTN_ERR_CUDA;
      // Every CTA of a problem streams its K and V.
      const int gq = attn::order_group(4.0 * D * avg_rows(pb.rows_k, pb), pb.problems);
      const unsigned gridq = static_cast<unsigned>(pb.problems) * static_cast<unsigned>(pb.qtiles);
      kq<<<gridq, 384, LQ::kAlloc, st>>>(mq, mk, mv, mdo, dvec, nlse2, static_cast<uint16_t*>(dq), pb.cu_q, pb.cu_k,
                                         pb.H, pb.rows_q, pb.rows_k, pb.bottom_right, scale, scale_log2, pb.problems,
                                         pb.qtiles, gq);
      if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    }
  }
  if (!DET && (phase == ATTN_BWD_ALL || phase == ATTN_BWD_CONVERT)) {
    const long long n8 = qrows * D / 8;
    long long post_blocks = (n8 + 255) / 256;
    if (post_blocks > 148LL * 16) post_blocks = 148LL * 16;
    attn::bwd_post_kernel<BF16>
        <<<static_cast<unsigned>(post_blocks), 256, 0, st>>>(dqacc, static_cast<uint16_t*>(dq), n8);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}


// The d = 256 backward: preprocess (no accumulator), the dK/dV kernel (one
// CTA per 64-key tile) and the dQ kernel (one CTA per query tile).  Always
// reproducible: no kernel adds into memory that another CTA writes.  K and V
// maps read 64-row boxes.
template <bool BF16, bool CAUSAL>
attn_status launch_bwd_wide(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const CUtensorMap& mdo, const void* o, const void* dout, const float* lse, void* dq,
                            void* dk, void* dv, float* ws, const Problem& pb, float scale, int phase, cudaStream_t st) {
  constexpr int D = 256;
  const WsLayout w = ws_layout(pb, D);
  float* dvec = ws + w.dvec;
  float* nlse2 = ws + w.nlse2;
  const float scale_log2 = scale * 1.4426950408889634f;
  if (phase == ATTN_BWD_ALL || phase == ATTN_BWD_PREPROCESS) {
    constexpr int kRowsPerBlock = 256 / (D / 8);
    const long long pre_blocks = (w.rows + kRowsPerBlock - 1) / kRowsPerBlock;
    attn::bwd_pre_kernel<D, BF16><<<static_cast<unsigned>(pre_blocks), 256, 0, st>>>(
        static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse, dvec, nlse2, nullptr, w.rows);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (phase == ATTN_BWD_ALL || phase == ATTN_BWD_MAIN) {
    using LK = attn::BwdKvWideLayout;
    auto kk = attn::bwd_kv_wide_kernel<BF16, CAUSAL>;
    if (set_smem(kk, LK::kAlloc) != cudaSuccess) return ATTN_ERR_CUDA;
    // Every CTA of a problem streams its Q and dO rows and their LSE and D.
    const int gk = attn::order_group((4.0 * D + 8.0) * avg_rows(pb.rows_q, pb), pb.problems);
    const int ktiles64 = 2 * pb.ktiles;  // 64-key tiles of the longest key sequence, at most
    const unsigned gridk = static_cast<unsigned>(pb.problems) * static_cast<unsigned>(ktiles64);
    kk<<<gridk, 384, LK::kAlloc, st>>>(mq, mk, mv, mdo, dvec, nlse2, static_cast<uint16_t*>(dk),
                                       static_cast<uint16_t*>(dv), pb.cu_q, pb.cu_k, pb.H, pb.rows_q, pb.rows_k,
                                       pb.bottom_right, scale, scale_log2, pb.problems, ktiles64, gk);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    using LQ = attn::BwdDqLayout<D>;
    auto kq = attn::bwd_dq_kernel<D, BF16, CAUSAL>;
    if (set_smem(kq, LQ::kAlloc) != cudaSuccess) return ATTN_ERR_CUDA;
    // Every CTA of a problem streams its K and V.
    const int gq = attn::order_group(4.0 * D * avg_rows(pb.rows_k, pb), pb.problems);
    const unsigned gridq = static_cast<unsigned>(pb.problems) * static_cast<unsigned>(pb.qtiles);
    kq<<<gridq, 384, LQ::kAlloc, st>>>(mq, mk, mv, mdo, dvec, nlse2, static_cast<uint16_t*>(dq), pb.cu_q, pb.cu_k,
                                       pb.H, pb.rows_q, pb.rows_k, pb.bottom_right, scale, scale_log2, pb.problems,
                                       pb.qtiles, gq);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;  // no dQ convert: the dQ kernel writes 16-bit dQ itself
}

template <int D, bool BF16>
attn_status dispatch_fwd_causal(int causal, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                const CUtensorMap& mo, void* o, float* lse, const Problem& pb, float sl2,
                                cudaStream_t st) {
  return causal ? launch_fwd<D, BF16, true>(mq, mk, mv, mo, o, lse, pb, sl2, st)
                : launch_fwd<D, BF16, false>(mq, mk, mv, mo, o, lse, pb, sl2, st);
}

// The forward launch shared by attn_fwd and attn_fwd_varlen.
attn_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, const Problem& pb, int d,
                     float scale, int causal, attn_dtype dtype, void* stream) {
  const bool bf16 = dtype == ATTN_BF16;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, q, pb.slabs, pb.rows_q, d, bf16) || !make_map(&mk, k, pb.slabs, pb.rows_k, d, bf16) ||
      !make_map(&mv, v, pb.slabs, pb.rows_k, d, bf16) || !make_map(&mo, o, pb.slabs, pb.rows_q, d, bf16))
    return ATTN_ERR_CUDA;
  const float sl2 = scale * 1.4426950408889634f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 64)
    return bf16 ? dispatch_fwd_causal<64, true>(causal, mq, mk, mv, mo, o, lse, pb, sl2, st)
                : dispatch_fwd_causal<64, false>(causal, mq, mk, mv, mo, o, lse, pb, sl2, st);
  if (d == 256)
    return bf16 ? dispatch_fwd_causal<256, true>(causal, mq, mk, mv, mo, o, lse, pb, sl2, st)
                : dispatch_fwd_causal<256, false>(causal, mq, mk, mv, mo, o, lse, pb, sl2, st);
  return bf16 ? dispatch_fwd_causal<128, true>(causal, mq, mk, mv, mo, o, lse, pb, sl2, st)
              : dispatch_fwd_causal<128, false>(causal, mq, mk, mv, mo, o, lse, pb, sl2, st);
}

// The FP8 forward launch shared by attn_fwd_fp8 and attn_fwd_fp8_varlen (d = 128).
attn_status fwd_fp8_impl(const void* q, const void* k, const void* v, void* o, float* lse, const Problem& pb,
                         float scale, float descale_q, float descale_k, float descale_v, int causal, void* stream) {
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, q, pb.slabs, pb.rows_q, 128, true, true) ||
      !make_map(&mk, k, pb.slabs, pb.rows_k, 128, true, true) ||
      !make_map(&mv, v, pb.slabs, pb.rows_k, 128, true, true) ||
      !make_map(&mo, o, pb.slabs, pb.rows_q, 128, true))  // O is bf16
    return ATTN_ERR_CUDA;
  // The scores are scale * (descale_q q) . (descale_k k): one factor, in log2 units.
  const float sl2 = scale * descale_q * descale_k * 1.4426950408889634f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return causal ? launch_fwd<128, true, true, true>(mq, mk, mv, mo, o, lse, pb, sl2, st, descale_v)
                : launch_fwd<128, true, false, true>(mq, mk, mv, mo, o, lse, pb, sl2, st, descale_v);
}

template <int D, bool BF16>
attn_status dispatch_bwd_causal(int causal, bool det, const CUtensorMap& mq, const CUtensorMap& mk,
                                const CUtensorMap& mv, const CUtensorMap& mdo, const void* o, const void* dout,
                                const float* lse, void* dq, void* dk, void* dv, float* ws, const Problem& pb,
                                float scale, int phase, cudaStream_t st) {
#define ATTN_LAUNCH_BWD(C, DT) \
  launch_bwd<D, BF16, C, DT>(mq, mk, mv, mdo, o, dout, lse, dq, dk, dv, ws, pb, scale, phase, st)
  if (det) return causal ? ATTN_LAUNCH_BWD(true, true) : ATTN_LAUNCH_BWD(false, true);
  return causal ? ATTN_LAUNCH_BWD(true, false) : ATTN_LAUNCH_BWD(false, false);
#undef ATTN_LAUNCH_BWD
}

// The backward launch shared by the dense and packed entry points.
attn_status bwd_launch(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dout, void* dq, void* dk, void* dv, void* workspace, const Problem& pb, int d,
                       float scale, int causal, attn_dtype dtype, int phase, bool det, void* stream) {
  const bool bf16 = dtype == ATTN_BF16;
  const int key_box = d == 256 ? 64 : kTile;  // the d = 256 kernels take 64-key tiles
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, q, pb.slabs, pb.rows_q, d, bf16) || !make_map(&mk, k, pb.slabs, pb.rows_k, d, bf16, false, key_box) ||
      !make_map(&mv, v, pb.slabs, pb.rows_k, d, bf16, false, key_box) ||
      !make_map(&mdo, dout, pb.slabs, pb.rows_q, d, bf16))
    return ATTN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  if (d == 256) {
    (void)det;  // always reproducible
#define ATTN_LAUNCH_WIDE(BB, C) \
  launch_bwd_wide<BB, C>(mq, mk, mv, mdo, o, dout, lse, dq, dk, dv, ws, pb, scale, phase, st)
    if (bf16) return causal ? ATTN_LAUNCH_WIDE(true, true) : ATTN_LAUNCH_WIDE(true, false);
    return causal ? ATTN_LAUNCH_WIDE(false, true) : ATTN_LAUNCH_WIDE(false, false);
#undef ATTN_LAUNCH_WIDE
  }
#define ATTN_DISPATCH_BWD(DD, BB) \
  dispatch_bwd_causal<DD, BB>(causal, det, mq, mk, mv, mdo, o, dout, lse, dq, dk, dv, ws, pb, scale, phase, st)
  if (d == 64) return bf16 ? ATTN_DISPATCH_BWD(64, true) : ATTN_DISPATCH_BWD(64, false);
  return bf16 ? ATTN_DISPATCH_BWD(128, true) : ATTN_DISPATCH_BWD(128, false);
#undef ATTN_DISPATCH_BWD
}

// The dense backward shared by attn_bwd_phase (det = false) and
// attn_bwd_deterministic (det = true).
attn_status bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, void* workspace, int B, int H, int Nq, int Nk, int d, float scale,
                     int causal, attn_dtype dtype, int phase, bool det, void* stream);

}  // namespace

// ------------------------------------------------ failure-detection self-test

namespace attn {

// One CTA of 64 threads.  Warp 0 waits, through the attention kernels' own
// bounded wait, on a barrier that nothing arrives on: it gives up after
// limit_ns, raises the CTA's abort flag and records the timeout.  Warp 1
// waits on a second such barrier with the kernels' 1 s limit and leaves
// through the abort flag as the other roles of an attention kernel would.
__global__ void __launch_bounds__(64) selftest_wait_kernel(unsigned long long limit_ns, int* result) {
  __shared__ uint64_t bars[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort = &abort_flag;
  bool ok;
  if (threadIdx.x < 32)
    ok = __all_sync(0xffffffffu, mbar_wait_for(&bars[0], 0, abort, limit_ns));
  else
    ok = __all_sync(0xffffffffu, mbar_wait(&bars[1], 0, abort));
  __syncthreads();
  if (threadIdx.x % 32 == 0) result[threadIdx.x / 32] = ok ? 1 : 0;
}

}  // namespace attn

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
  attn::TraceRange trace("attn_fwd");
  const attn_status cs = check_common(B, H, Nq, Nk, d, causal, dtype);
  if (cs != ATTN_OK) return cs;
  if (B == 0 || H == 0 || Nq == 0) return ATTN_OK;  // no query rows: nothing to write
  if (Nk == 0) return ATTN_ERR_INVALID_ARG;         // a softmax over no keys is undefined
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, o, lse, dense_problem(B, H, Nq, Nk, causal), d, scale, causal, dtype, stream);
}

attn_status attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                         int Nk, int d, float scale, float descale_q, float descale_k, float descale_v, int causal,
                         void* stream) {
  attn::TraceRange trace("attn_fwd_fp8");
  const attn_status cs = check_common(B, H, Nq, Nk, d, causal, ATTN_BF16);
  if (cs != ATTN_OK) return cs;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!std::isfinite(descale_q) || !std::isfinite(descale_k) || !std::isfinite(descale_v) || !std::isfinite(scale))
    return ATTN_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || Nq == 0) return ATTN_OK;  // no query rows: nothing to write
  if (Nk == 0) return ATTN_ERR_INVALID_ARG;         // a softmax over no keys is undefined
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_INVALID_ARG;
  return fwd_fp8_impl(q, k, v, o, lse, dense_problem(B, H, Nq, Nk, causal), scale, descale_q, descale_k, descale_v,
                      causal, stream);
}

attn_status attn_fwd_fp8_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                                const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H, int total_q,
                                int total_k, int max_seqlen_q, int max_seqlen_k, int d, float scale, float descale_q,
                                float descale_k, float descale_v, int causal, void* stream) {
  attn::TraceRange trace("attn_fwd_fp8_varlen");
  const attn_status cs = check_varlen(B, H, total_q, total_k, max_seqlen_q, max_seqlen_k, d, causal, ATTN_BF16);
  if (cs != ATTN_OK) return cs;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!std::isfinite(descale_q) || !std::isfinite(descale_k) || !std::isfinite(descale_v) || !std::isfinite(scale))
    return ATTN_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || total_q == 0 || max_seqlen_q == 0) return ATTN_OK;  // no query rows
  if (!q || !k || !v || !o || !lse || !cu_seqlens_q || !cu_seqlens_k) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (total_k == 0)  // no sequence has keys: O = 0, LSE = -inf (the query tensor stands in for K and V)
    return fwd_fp8_impl(q, q, q, o, lse,
                        varlen_problem(B, H, total_q, 1, max_seqlen_q, 1, cu_seqlens_q, cu_seqlens_k, causal), scale,
                        descale_q, descale_k, descale_v, causal, stream);
  return fwd_fp8_impl(q, k, v, o, lse,
                      varlen_problem(B, H, total_q, total_k, max_seqlen_q, max_seqlen_k, cu_seqlens_q, cu_seqlens_k,
                                     causal),
                      scale, descale_q, descale_k, descale_v, causal, stream);
}

attn_status attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens_q,
                            const int* cu_seqlens_k, int B, int H, int total_q, int total_k, int max_seqlen_q,
                            int max_seqlen_k, int d, float scale, int causal, attn_dtype dtype, void* stream) {
  attn::TraceRange trace("attn_fwd_varlen");
  const attn_status cs = check_varlen(B, H, total_q, total_k, max_seqlen_q, max_seqlen_k, d, causal, dtype);
  if (cs != ATTN_OK) return cs;
  if (B == 0 || H == 0 || total_q == 0 || max_seqlen_q == 0) return ATTN_OK;  // no query rows
  if (!q || !k || !v || !o || !lse || !cu_seqlens_q || !cu_seqlens_k) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (total_k == 0) {  // no sequence has keys: every row's softmax is empty (O = 0, LSE = -inf)
    // The kernels write exactly that when they find no key tile; they need a
    // valid K/V map, so give them the query tensor as a stand-in of one row.
    return fwd_impl(q, q, q, o, lse, varlen_problem(B, H, total_q, 1, max_seqlen_q, 1, cu_seqlens_q, cu_seqlens_k,
                                                    causal), d, scale, causal, dtype, stream);
  }
  return fwd_impl(q, k, v, o, lse,
                  varlen_problem(B, H, total_q, total_k, max_seqlen_q, max_seqlen_k, cu_seqlens_q, cu_seqlens_k,
                                 causal),
                  d, scale, causal, dtype, stream);
}

size_t attn_bwd_workspace_bytes(int B, int H, int Nq, int Nk, int d) {
  if (B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return 0;  // empty problems need none
  const long long bh = static_cast<long long>(B) * H;
  if (bh > 0x7fffffffLL || bh * Nq > (1LL << 40)) return 0;
  return static_cast<size_t>(ws_layout(dense_problem(B, H, Nq, Nk, 0), d).words * 4);
}

size_t attn_bwd_varlen_workspace_bytes(int B, int H, int total_q, int max_seqlen_q, int d) {
  if (B <= 0 || H <= 0 || total_q <= 0 || max_seqlen_q <= 0 || d <= 0) return 0;
  if (static_cast<long long>(B) * H > 0x7fffffffLL || static_cast<long long>(H) * total_q > (1LL << 40)) return 0;
  return static_cast<size_t>(
      ws_layout(varlen_problem(B, H, total_q, 1, max_seqlen_q, 1, nullptr, nullptr, 0), d).words * 4);
}

attn_status attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* dout, void* dq, void* dk, void* dv, void* workspace, const int* cu_seqlens_q,
                            const int* cu_seqlens_k, int B, int H, int total_q, int total_k, int max_seqlen_q,
                            int max_seqlen_k, int d, float scale, int causal, attn_dtype dtype, int deterministic,
                            void* stream) {
  attn::TraceRange trace("attn_bwd_varlen");
  const attn_status cs = check_varlen(B, H, total_q, total_k, max_seqlen_q, max_seqlen_k, d, causal, dtype);
  if (cs != ATTN_OK) return cs;
  if (B == 0 || H == 0) return ATTN_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (total_q == 0 || max_seqlen_q == 0) {  // no query rows: dK = dV = 0
    const size_t bytes = static_cast<size_t>(H) * total_k * d * 2;
    if (bytes == 0) return ATTN_OK;
    if (!dk || !dv) return ATTN_ERR_INVALID_ARG;
    if (cudaMemsetAsync(dk, 0, bytes, st) != cudaSuccess || cudaMemsetAsync(dv, 0, bytes, st) != cudaSuccess)
      return ATTN_ERR_CUDA;
    return ATTN_OK;
  }
  if (total_k == 0) {  // no key rows: every softmax is empty, so dQ = 0
    if (!dq) return ATTN_ERR_INVALID_ARG;
    return cudaMemsetAsync(dq, 0, static_cast<size_t>(H) * total_q * d * 2, st) == cudaSuccess ? ATTN_OK
                                                                                                 : ATTN_ERR_CUDA;
  }
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace || !cu_seqlens_q || !cu_seqlens_k)
    return ATTN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return ATTN_ERR_INVALID_ARG;
  return bwd_launch(q, k, v, o, lse, dout, dq, dk, dv, workspace,
                    varlen_problem(B, H, total_q, total_k, max_seqlen_q, max_seqlen_k, cu_seqlens_q, cu_seqlens_k,
                                   causal),
                    d, scale, causal, dtype, ATTN_BWD_ALL, deterministic != 0, stream);
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
  attn::TraceRange trace(det ? "attn_bwd_deterministic" : "attn_bwd");
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
  return bwd_launch(q, k, v, o, lse, dout, dq, dk, dv, workspace, dense_problem(B, H, Nq, Nk, causal), d, scale,
                    causal, dtype, phase, det, stream);
}

}  // namespace

extern "C" {

attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                             const void* dout, void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int d,
                             float scale, int causal, attn_dtype dtype, void* stream) {
  attn::TraceRange trace("attn_bwd_noalloc");
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

attn_status attn_selftest_wait_timeout(int limit_us, int* result, void* stream) {
  attn::TraceRange trace("attn_selftest_wait_timeout");
  if (limit_us < 1 || limit_us > 1000000 || !result) return ATTN_ERR_INVALID_ARG;
  attn::selftest_wait_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_us) * 1000ull, result);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

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
    case ATTN_ERR_RANGE: return "fp16 backward: a per-query term |LSE/scale| or |D| reached 2^31";
  }
  return "unknown status";
}

}  // extern "C"
