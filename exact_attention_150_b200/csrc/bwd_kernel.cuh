// bwd_kernel.cuh -- attention backward for sm_100a, by recomputation.
//
// The attention matrix is not stored by the forward pass; the backward pass
// recomputes it from Q, K and the saved row log-sum-exp (page "FlashAttention
// 核心原理", part 2 item 3).  Three kernels:
//
//   bwd_pre_kernel    D_i = sum_c dO_ic O_ic, -log2(e) * LSE_i, and dQacc = 0
//   bwd_main_kernel   one CTA per (key tile j, problem), a problem being one
//                     (batch, head) slice or one sequence of one head of a
//                     packed variable-length batch: K_j, V_j stay in
//                     shared memory; for every query tile i that sees them
//                       S'^T  = K_j Q_i^T - LSE_i / scale   (tcgen05, TMEM)
//                       dP'^T = V_j dO_i^T - D_i            (tcgen05, TMEM)
//                       P^T   = exp2(S'^T * scale * log2e)
//                       dS^T  = P^T * dP'^T
//                       dV_j += P^T dO_i              (A = P^T from TMEM)
//                       dK_j += dS^T Q_i              (A = dS^T from TMEM)
//                       dQacc_i += scale * dS K_j     (fp32 atomics)
//                     then dK_j = scale * dK_j and dV_j are written once.
//                     (dQ is formed transposed, dQ^T = K_j^T dS^T, when
//                     d = 128, so that the atomics of a warp cover one
//                     contiguous 128-byte row segment.)
//   bwd_post_kernel   dQ = 16-bit(dQacc)
//
// Main-kernel CTA layout (512 threads, one CTA per SM):
//   warp 0       TMA producer (K_j, V_j once; Q_i, dO_i through 2 stages)
//   warp 1       MMA issuer (one thread)
//   warp 2       TMEM allocation
//   warps 4-7    P / dS for query columns [0, 64)   (thread = key row = TMEM lane)
//   warps 8-11   P / dS for query columns [64, 128)
//   warps 12-15  dQ drain, then the dK/dV epilogue
// Tensor memory (d = 128):
//   [0,128)    S^T fp32; overwritten in place by P^T (16-bit pairs) in
//              [0,32) and [64,96)
//   [128,256)  dP^T fp32, then dS^T packed 16-bit over it, then
//              dQ^T = K^T dS^T fp32 (lane = head-dim index)
//   [256,384)  dV,  [384,512) dK
// For d = 64 the dQ tile is dS K (lane = query row) in [128,192), dV in
// [256,320) and dK in [320,384).
// The dS pass writes dS^T twice: packed 16-bit over dP^T in TMEM, the A
// operand of dK += dS^T Q (a TS product, which reads only Q from shared
// memory), and 128-byte swizzled into shared memory ([key][query]), the
// MN-major operand of the dQ product, which then overwrites the dP^T
// columns (the tensor core runs dK first).  S^T lives in its own columns,
// so the next query tile's S^T is issued right after dV, and per query tile
// the MMA issue order is
//   dP^T, dV, S^T(next), dK, dQ
// while the softmax warps go from this tile's dS pass straight to the next
// tile's P pass as dK and dQ run on the tensor core.
// The per-query terms -LSE_i / scale and -D_i enter through one extra K step
// of 16 in the S^T and dP^T products: the A operand is a constant tile that
// selects them ([w0,w1,w2,w3,0,...] or [0,0,0,0,w0,w1,w2,w3,0,...] in every
// key row) and the B operand holds, per query row, each term as four 16-bit
// pieces whose weighted sum is the term (see ext_pieces).  The softmax warps
// thus need no per-query data at all.
// Warp 3 writes that B block for the next query tile while the current one
// is in use (single buffer, released by the dP^T product).
#pragma once

#include "sm100.cuh"
#include "tile_order.h"

namespace attn {

constexpr int kBwdTile = 128;

template <int D>
struct BwdLayout {
  static constexpr int kChunkBytes = kBwdTile * 128;
  static constexpr int kTileBytes = kBwdTile * D * 2;
  static constexpr int kStages = 2;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kStageOff = 2 * kTileBytes;  // stage s: Q at +s*2T, dO at +s*2T+T
  static constexpr int kDSOff = kStageOff + kStages * 2 * kTileBytes;
  static constexpr int kDSBytes = kBwdTile * kBwdTile * 2;
  // Extra K step: A_ext = two unswizzled 8x16-byte core matrices per term
  // (selector row, zeros), read with a zero row-group stride; B_ext = 128
  // query rows x 16 bytes [s0, s1, s2, s3, d0, d1, d2, d3].
  static constexpr int kAExtOff = kDSOff + kDSBytes;
  static constexpr int kAExtBytes = 4 * 128;
  static constexpr int kBExtOff = kAExtOff + kAExtBytes;
  static constexpr int kBExtBytes = kBwdTile * 16;
  static constexpr int kBarOff = kBExtOff + kBExtBytes;
  // kv_full, qd_full[S], qd_empty[S], s_full, dp_full, p_full, ds_full, dq_full, dq_free, acc_full, mma_done,
  // bext_full, bext_free
  static constexpr int kNumBars = 1 + 2 * kStages + 10;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  // The tiles need a 1024-byte aligned base.  The dynamic shared window
  // starts 1024-byte aligned in practice; the slack below covers what the
  // 227 KB limit leaves, and the kernel checks the real need at entry.
  static constexpr int kAlloc = kBytes + 1024 <= 232448 ? kBytes + 1024 : 232448;
  static_assert(kBytes <= 232448, "shared memory budget");
};

// One group of D/8 threads per row; each thread handles 8 elements.
template <int D, bool BF16>
__global__ void __launch_bounds__(256)
    bwd_pre_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                   const float* __restrict__ lse, float* __restrict__ dvec, float* __restrict__ nlse2,
                   float* __restrict__ dqacc, long long rows) {
  constexpr int kTpr = D / 8;
  constexpr int kRowsPerBlock = 256 / kTpr;
  const long long row = static_cast<long long>(blockIdx.x) * kRowsPerBlock + threadIdx.x / kTpr;
  const int seg = threadIdx.x % kTpr;
  float acc = 0.f;
  if (row < rows) {
    const size_t off = static_cast<size_t>(row) * D + seg * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(o + off);
    const uint4 b = *reinterpret_cast<const uint4*>(dout + off);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w};
    const uint32_t bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = unpack2<BF16>(av[i]);
      const float2 y = unpack2<BF16>(bv[i]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
    if (dqacc != nullptr) {  // the atomic-dQ backward accumulates into it
      float4* z = reinterpret_cast<float4*>(dqacc + off);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int m = kTpr / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if (row < rows && seg == 0) {
    dvec[row] = acc;
    // A row that sees no key (LSE = -inf) has every P masked; a finite
    // stand-in keeps the extra MMA K step free of inf - inf.
    nlse2[row] = lse[row] == -INFINITY ? 0.f : -lse[row] * 1.4426950408889634074f;
  }
}

// Weight of piece i of a per-query term in the extra K step.  bf16 has
// fp32's exponent range: three pieces of weight 1 (v = b0 + b1 + b2, the
// remainder of each rounding carried by the next, 24 bits in all).  fp16 tops
// out at 65504, so its four pieces sit on a ladder of powers of two 11 bits
// apart, each holding what the one above left:
//   v = 2^15 b0 + 2^5 b1 + 2^-6 b2 + 2^-14 b3,
// exact to about 2^-28 and valid for |v| < 2^31 (b0 <= 65504).  Every weight
// is a 16-bit normal number, and every product with it is exact in fp32.
template <bool BF16>
__device__ __forceinline__ float ext_weight(int i) {
  if constexpr (BF16) return i < 3 ? 1.f : 0.f;
  return i == 0 ? 32768.f : (i == 1 ? 32.f : (i == 2 ? 0.015625f : 6.103515625e-05f));
}
// 1 / ext_weight(i), exact (powers of two).
template <bool BF16>
__device__ __forceinline__ float ext_inv_weight(int i) {
  if constexpr (BF16) return 1.f;
  return i == 0 ? 3.0517578125e-05f : (i == 1 ? 0.03125f : (i == 2 ? 64.f : 16384.f));
}
// Largest |v| the pieces represent: 2^31 for fp16; bf16 covers every finite
// fp32 value.
template <bool BF16>
__device__ __forceinline__ bool ext_in_range(float v) {
  if constexpr (BF16) return fabsf(v) <= 3.0e38f;
  return fabsf(v) < 2147483648.0f;
}

// The four 16-bit pieces of v, packed [b0 | b1], [b2 | b3].  Each piece is
// the 16-bit rounding of the remainder scaled by 1 / weight; an fp16 piece
// that would be subnormal is set to 0 and its value left to the pieces below,
// so the result never depends on how the tensor core treats subnormals.  The
// remainder updates are exact (Sterbenz: the subtracted value is within a
// factor 2 of the remainder).
template <bool BF16>
__device__ __forceinline__ uint2 ext_pieces(float v) {
  float b[4];
  float r = v;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (BF16 && i == 3) {
      b[i] = 0.f;
      continue;
    }
    float x = unpack2<BF16>(pack2<BF16>(r * ext_inv_weight<BF16>(i), 0.f)).x;
    if (!BF16 && fabsf(x) < 6.103515625e-05f) x = 0.f;
    b[i] = x;
    r -= x * ext_weight<BF16>(i);
  }
  return make_uint2(pack2<BF16>(b[0], b[1]), pack2<BF16>(b[2], b[3]));
}

template <bool BF16>
__global__ void __launch_bounds__(256)
    bwd_post_kernel(const float* __restrict__ dqacc, uint16_t* __restrict__ dq, long long n8) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(dqacc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(dqacc)[2 * i + 1];
    reinterpret_cast<uint4*>(dq)[i] =
        make_uint4(pack2<BF16>(a.x, a.y), pack2<BF16>(a.z, a.w), pack2<BF16>(b.x, b.y), pack2<BF16>(b.z, b.w));
  }
}

// DQ = true: the dQ contributions are formed here and added into the fp32
// accumulator with atomics.  DQ = false: this kernel writes dK and dV only,
// and bwd_dq_kernel computes dQ on its own (the reproducible backward).
// max_qtiles: query tiles of the longest sequence (packed batches).
template <int D, bool BF16, bool CAUSAL, bool DQ>
__global__ void __launch_bounds__(512, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const float* __restrict__ dvec, const float* __restrict__ nlse2, float* __restrict__ dqacc,
                    uint16_t* __restrict__ dk_ptr, uint16_t* __restrict__ dv_ptr, const int* __restrict__ cu_q,
                    const int* __restrict__ cu_k, int H, int Nq, int Nk, int bottom_right, int max_qtiles,
                    float scale, float scale_log2, int problems, int grid_tiles, int group) {
  using L = BwdLayout<D>;
  constexpr bool kDqT = (D == 128);  // dQ formed transposed (see above)
  constexpr uint32_t kColDP = 128, kColDQ = 128, kColDV = 256, kColDK = 256 + D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kv_full = bars;
  uint64_t* qd_full = bars + 1;
  uint64_t* qd_empty = qd_full + L::kStages;
  uint64_t* s_full = qd_empty + L::kStages;
  uint64_t* dp_full = s_full + 1;
  uint64_t* p_full = s_full + 2;
  uint64_t* ds_full = s_full + 3;
  uint64_t* dq_full = s_full + 4;
  uint64_t* dq_free = s_full + 5;
  uint64_t* acc_full = s_full + 6;
  uint64_t* mma_done = s_full + 7;
  uint64_t* bext_full = s_full + 8;  // warp 3 -> MMA: B_ext holds the current tile's terms
  uint64_t* bext_free = s_full + 9;  // MMA -> warp 3: the dP^T product has read B_ext
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // The problem of this CTA: slab z of the tensor maps ([z][Nq or Nk][D])
  // and rows [q0, q0 + nq) / [k0, k0 + nk) of it (one slab per (batch,
  // head) for dense batches; one per head for packed variable-length
  // batches, sequence b's rows from the offsets clamped to the slab).
  // The grid is one-dimensional, in the grouped launch order of
  // tile_order.h: px is the problem, j the key tile.
  int px, j;
  grouped_order(blockIdx.x, problems, grid_tiles, group, &px, &j);
  int z = px, q0 = 0, k0 = 0, nq = Nq, nk = Nk;
  if (cu_q != nullptr) {
    const int b = px / H;
    z = px - b * H;
    auto clamp = [](int v, int hi) { return v < 0 ? 0 : (v > hi ? hi : v); };
    q0 = clamp(cu_q[b], Nq);
    k0 = clamp(cu_k[b], Nk);
    nq = clamp(cu_q[b + 1], Nq) - q0;
    nk = clamp(cu_k[b + 1], Nk) - k0;
    nq = nq < 0 ? 0 : nq;
    nk = nk < 0 ? 0 : nk;
    // Rows past max_seqlen_q (the grid's query tiles) are not computed.
    nq = nq < max_qtiles * kBwdTile ? nq : max_qtiles * kBwdTile;
  }
  // Key tile j; causal: small j has the most work and launches first.
  if (j * kBwdTile >= nk) return;  // a sequence shorter than the grid
  const int nqt = (nq + kBwdTile - 1) / kBwdTile;  // the last tiles may be ragged
  // Causal: query q sees key k iff k <= q + off (off = 0 top-left,
  // nk - nq bottom-right); the first query tile that sees key j * 128 is
  // the one holding query j * 128 - off.
  const int off = bottom_right ? nk - nq : 0;
  const int first_q = j * kBwdTile - off;
  const int i0 = CAUSAL ? (first_q > 0 ? first_q / kBwdTile : 0) : 0;
  const int n_it = nqt - i0;
  const int kv_valid = nk - j * kBwdTile < kBwdTile ? nk - j * kBwdTile : kBwdTile;  // key rows of this tile
  const size_t krow0 = static_cast<size_t>(z) * Nk + k0 + static_cast<size_t>(j) * kBwdTile;  // first key row
  const size_t qslab = static_cast<size_t>(z) * Nq + q0;  // row of this sequence's first query

  if (n_it <= 0) {
    // No query sees these keys (causal with more keys than queries, or a
    // sequence without queries): their gradients are zero.
    const int n16 = kv_valid * D / 8;
    const size_t base = krow0 * D / 8;
    for (int e = threadIdx.x; e < n16; e += blockDim.x) {
      reinterpret_cast<uint4*>(dk_ptr)[base + e] = make_uint4(0u, 0u, 0u, 0u);
      reinterpret_cast<uint4*>(dv_ptr)[base + e] = make_uint4(0u, 0u, 0u, 0u);
    }
    return;
  }

  // Refuse to run (and report) if alignment left too little shared memory.
  if (static_cast<uint32_t>(smem - smem_raw) + L::kBytes > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) atomicExch(&g_device_status, kStatusSmem);
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&qd_full[s], 1);
      mbar_init(&qd_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 256);
    mbar_init(ds_full, 256);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(acc_full, 1);
    mbar_init(mma_done, 1);
    mbar_init(bext_full, 32);
    mbar_init(bext_free, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 3) {
    // A_ext: [sel_s: rows of w0,w1,w2,w3,0,..] [zeros] [sel_d: rows of 0,0,0,0,w0,w1,w2,w3] [zeros]
    // (the piece weights of ext_pieces).
    uint32_t* a = reinterpret_cast<uint32_t*>(smem + L::kAExtOff);
    for (int i = lane; i < L::kAExtBytes / 4; i += 32) {
      const int cm = i / 32, w = i % 4;  // core matrix, 32-bit word within a 16-byte row
      const bool sel = (cm == 0 && w < 2) || (cm == 2 && w >= 2);
      const int p = 2 * (w & 1);          // first piece of this word
      a[i] = sel ? pack2<BF16>(ext_weight<BF16>(p), ext_weight<BF16>(p + 1)) : 0u;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(kv_full, 2 * L::kTileBytes);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + L::kKOff + c * L::kChunkBytes, &tm_k, kv_full, c * 64, k0 + j * kBwdTile, z);
        tma_load_3d(smem + L::kVOff + c * L::kChunkBytes, &tm_v, kv_full, c * 64, k0 + j * kBwdTile, z);
      }
      int it = 0;
      bool ok = true;
      for (; it < n_it; ++it) {
        const int s = it % L::kStages;
        const uint32_t ph = (it / L::kStages) & 1;
        if (!mbar_wait(&qd_empty[s], ph ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        const int qrow = q0 + (i0 + it) * kBwdTile;
        mbar_arrive_expect_tx(&qd_full[s], 2 * L::kTileBytes);
        uint8_t* qdst = smem + L::kStageOff + s * 2 * L::kTileBytes;
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(qdst + c * L::kChunkBytes, &tm_q, &qd_full[s], c * 64, qrow, z);
          tma_load_3d(qdst + L::kTileBytes + c * L::kChunkBytes, &tm_do, &qd_full[s], c * 64, qrow, z);
        }
      }
      if (!ok) {
        mbar_drain(kv_full, 0);
        const int first = it > L::kStages ? it - L::kStages : 0;
        for (int i = first; i < it; ++i) mbar_drain(&qd_full[i % L::kStages], (i / L::kStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (descriptors stay warp-uniform); one
    // elected lane issues each group of MMAs together with its commits.
    constexpr uint32_t kIdS = idesc_f16(BF16, 128, 128, false, false);  // K-major x K-major
    constexpr uint32_t kIdAcc = idesc_f16(BF16, 128, D, false, true);   // K-major A x MN-major B
    // dQ^T = K^T dS^T (M = d) or dQ = dS K (M = queries); both operands MN-major.
    constexpr uint32_t kIdQ = kDqT ? idesc_f16(BF16, 128, 128, true, true) : idesc_f16(BF16, 128, 64, true, true);
    const uint32_t k_addr = smem_u32(smem + L::kKOff);
    const uint32_t v_addr = smem_u32(smem + L::kVOff);
    const uint32_t ds_addr = smem_u32(smem + L::kDSOff);
    // K-major SW128 operands step 32 bytes per K step inside a 128-byte row
    // and 16 KB per 64-column chunk; MN-major ones step 16 rows (2048 bytes).
    auto kmaj = [](int ks) { return static_cast<uint64_t>(((ks >> 2) * L::kChunkBytes + (ks & 3) * 32) >> 4); };
    const uint64_t kd_k = sdesc_sw128(k_addr, 16, 1024), kd_v = sdesc_sw128(v_addr, 16, 1024);
    const uint64_t mn_k = sdesc_sw128(k_addr, L::kChunkBytes, 1024), mn_ds = sdesc_sw128(ds_addr, L::kChunkBytes, 1024);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    auto stage_addr = [&](int it) {
      return smem_u32(smem + L::kStageOff + (it % L::kStages) * 2 * L::kTileBytes);
    };
    // Packed 16-bit P^T columns of K step ks (16 queries).
    auto p_col = [](int ks) { return static_cast<uint32_t>(64 * (ks >> 2) + 8 * (ks & 3)); };
    // Extra K step: A_ext selects a term (zero row-group stride: one core
    // matrix serves all 128 rows), B_ext holds it per query row.
    const uint64_t ext_s = sdesc_noswz(smem_u32(smem + L::kAExtOff), 128, 0);
    const uint64_t ext_d = sdesc_noswz(smem_u32(smem + L::kAExtOff + 256), 128, 0);
    const uint64_t ext_b = sdesc_noswz(smem_u32(smem + L::kBExtOff), 0, 128);
    const bool zero_scale = scale == 0.f;  // then S' is the LSE term alone
    auto issue_st = [&](uint32_t q_addr) {
      const uint64_t qd = sdesc_sw128(q_addr, 16, 1024);
      if (!zero_scale) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) mma_ss(tmem, kd_k + kmaj(ks), qd + kmaj(ks), kIdS, ks > 0 ? 1u : 0u);
      }
      mma_ss(tmem, ext_s, ext_b, kIdS, zero_scale ? 0u : 1u);
    };
    auto issue_dp = [&](int it) {  // dP'^T of query tile it, then its commits
      const uint64_t dod_k = sdesc_sw128(stage_addr(it) + L::kTileBytes, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        mma_ss(tmem + kColDP, kd_v + kmaj(ks), dod_k + kmaj(ks), kIdS, ks > 0 ? 1u : 0u);
      mma_ss(tmem + kColDP, ext_d, ext_b, kIdS, 1u);
      mma_commit(dp_full);
      mma_commit(bext_free);  // S^T and dP^T of this tile have read B_ext
    };
    // Issue order per query tile it (DQ): dP^T(it) once the dQ drain has
    // read the columns it reuses, dV(it), S^T(it+1), dK(it), dQ(it).
    // Without dQ, dS^T is only the A operand of dK, so the dS pass writes it
    // over dP^T in tensor memory (no shared-memory copy) and dK reads it
    // from there:  dV(it), S^T(it+1), dK(it), dP^T(it+1).
    bool ok = wait_all(kv_full, 0) && wait_all(&qd_full[0], 0) && wait_all(bext_full, 0);
    if (ok && n_it > 0) {
      tc_fence_after();
      if (elect_one()) {
        issue_st(stage_addr(0));
        mma_commit(s_full);
        if constexpr (!DQ) issue_dp(0);
      }
      __syncwarp();
    }
    for (int it = 0; ok && it < n_it; ++it) {
      const uint32_t q_addr = stage_addr(it);
      const uint32_t do_addr = q_addr + L::kTileBytes;
      const uint64_t dod_mn = sdesc_sw128(do_addr, L::kChunkBytes, 1024);
      const uint64_t qd_mn = sdesc_sw128(q_addr, L::kChunkBytes, 1024);
      if constexpr (DQ) {
        // dP^T overwrites the previous tile's dQ columns: wait for the drain.
        if (it > 0 && !(ok = wait_all(dq_free, (it - 1) & 1))) break;
        tc_fence_after();
        if (elect_one()) issue_dp(it);
        __syncwarp();
      }
      if (!(ok = wait_all(p_full, it & 1))) break;
      tc_fence_after();
      if (elect_one()) {
        // dV += P^T dO: A from TMEM, B = dO MN-major (16 query rows per K step).
#pragma unroll
        for (int ks = 0; ks < kBwdTile / 16; ++ks)
          mma_ts(tmem + kColDV, tmem + p_col(ks), dod_mn + 128 * ks, kIdAcc, (it > 0 || ks > 0) ? 1u : 0u);
      }
      __syncwarp();
      // The next tile's S^T only overwrites P^T, which dV (issued above)
      // consumes first; issuing it now lets the softmax warps move on to
      // the next P pass as soon as this tile's dS pass is done.
      if (it + 1 < n_it) {
        if (!(ok = wait_all(&qd_full[(it + 1) % L::kStages], ((it + 1) / L::kStages) & 1))) break;
        if (!(ok = wait_all(bext_full, (it + 1) & 1))) break;
        tc_fence_after();
        if (elect_one()) {
          issue_st(stage_addr(it + 1));
          mma_commit(s_full);
        }
        __syncwarp();
      }
      if (!(ok = wait_all(ds_full, it & 1))) break;
      tc_fence_after();
      if (elect_one()) {
        // dK += dS^T Q: A = dS^T packed over dP^T in tensor memory, B = Q
        // MN-major.
#pragma unroll
        for (int ks = 0; ks < kBwdTile / 16; ++ks) {
          mma_ts(tmem + kColDK, tmem + kColDP + p_col(ks), qd_mn + 128 * ks, kIdAcc, (it > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&qd_empty[it % L::kStages]);
        if (it == n_it - 1) mma_commit(acc_full);
        if constexpr (!DQ) {
          if (it + 1 < n_it) issue_dp(it + 1);  // over dS^T(it), which dK (issued above) reads first
        }
        if constexpr (DQ) {
#pragma unroll
          for (int ks = 0; ks < kBwdTile / 16; ++ks) {
            if constexpr (kDqT)  // A = K^T (M = d), B = dS^T (N = queries)
              mma_ss(tmem + kColDQ, mn_k + 128 * ks, mn_ds + 128 * ks, kIdQ, ks > 0 ? 1u : 0u);
            else  // A = dS (M = queries), B = K (N = d)
              mma_ss(tmem + kColDQ, mn_ds + 128 * ks, mn_k + 128 * ks, kIdQ, ks > 0 ? 1u : 0u);
          }
          mma_commit(dq_full);
        }
      }
      __syncwarp();
    }
    if (elect_one()) mma_commit(mma_done);
    __syncwarp();
    mbar_drain(mma_done, 0);
  } else if (warp == 3) {
    // ------------------------------------------------------------ B_ext writer
    // Row q of B_ext: [s0, s1, s2, s3, d0, d1, d2, d3], the 16-bit pieces
    // (ext_pieces) of s = -LSE_q / scale (-log2(e) LSE_q when scale == 0)
    // and d = -D_q.  A term outside the pieces' range (fp16: |LSE_q / scale|
    // or |D_q| >= 2^31) is recorded as ATTN_ERR_RANGE in the device status
    // word; its pieces are then zero rather than infinite, so the products
    // stay finite.
    const float inv_c = scale == 0.f ? 1.f : 1.f / scale_log2;  // nlse2 = -log2(e) LSE
    uint4* bext = reinterpret_cast<uint4*>(smem + L::kBExtOff);
    bool range_ok = true;
    for (int it = 0; it < n_it; ++it) {
      const size_t vbase = qslab + static_cast<size_t>(i0 + it) * kBwdTile;
      const int q_valid = nq - (i0 + it) * kBwdTile;
      float sv[4], dv4[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const bool in = lane + 32 * k < q_valid;  // rows past the sequence: zeros (their P is masked)
        sv[k] = in ? nlse2[vbase + lane + 32 * k] * inv_c : 0.f;
        dv4[k] = in ? -dvec[vbase + lane + 32 * k] : 0.f;
        if (!ext_in_range<BF16>(sv[k]) || !ext_in_range<BF16>(dv4[k])) {
          range_ok = false;
          sv[k] = ext_in_range<BF16>(sv[k]) ? sv[k] : 0.f;
          dv4[k] = ext_in_range<BF16>(dv4[k]) ? dv4[k] : 0.f;
        }
      }
      if (it > 0 && !__all_sync(0xffffffffu, mbar_wait(bext_free, (it - 1) & 1, abort_flag))) break;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint2 s4 = ext_pieces<BF16>(sv[k]), d4 = ext_pieces<BF16>(dv4[k]);
        bext[lane + 32 * k] = make_uint4(s4.x, s4.y, d4.x, d4.y);
      }
      fence_proxy_async_smem();
      mbar_arrive(bext_full);
    }
    if (!__all_sync(0xffffffffu, range_ok) && lane == 0) atomicExch(&g_device_status, kStatusRange);
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ P and dS
    const int h = (warp - 4) >> 2;  // query columns [64h, 64h + 64)
    const int wq = warp & 3;
    const int r = wq * 32 + lane;   // key row within tile j = TMEM lane
    const float cs = scale == 0.f ? 1.f : scale_log2;  // S' is in units of 1 / scale
    const float2 cs2 = make_float2(cs, cs);
    const uint32_t t_row = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    uint8_t* ds_row = smem + L::kDSOff + h * L::kChunkBytes + r * 128;
    for (int it = 0; it < n_it; ++it) {
      const int i = i0 + it;
      // Key row r sees query q of this tile iff q >= dlt + r; the tile needs
      // the causal test if its last key row does not see query 0.
      const int dlt = (j - i) * kBwdTile - off;
      const bool diag = CAUSAL && dlt + kBwdTile - 1 > 0;
      // Key row r sees query columns [lo, hi) of this tile: lo from the
      // causal mask, hi = the queries before Nq, and none at all if the key
      // is past Nk.  P is zeroed outside.
      const int q_valid = nq - i * kBwdTile;
      const bool masked = diag || kv_valid < kBwdTile || q_valid < kBwdTile;
      const int lo = diag && dlt + r > 0 ? dlt + r : 0;
      const int hi = r < kv_valid ? (q_valid < kBwdTile ? q_valid : kBwdTile) : 0;
      const uint32_t span = hi > lo ? static_cast<uint32_t>(hi - lo) : 0u;
      const int q_base = 64 * h - lo;  // column q tests (q - lo) < span, unsigned
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, it & 1, abort_flag))) break;
      tc_fence_after();
      // P pass: P^T = exp2(S'^T * scale * log2e), packed 16-bit.
      uint32_t ppk[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sr[32];
        tmem_ld32(t_row + 64 * h + 32 * c, sr);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const int x = 16 * g + e;
            const float2 a = mul2(make_float2(__uint_as_float(sr[x]), __uint_as_float(sr[x + 1])), cs2);
            float p0 = ex2(a.x);
            float p1 = ex2(a.y);
            if (masked) {
              const int q = q_base + 32 * c + x;
              if (static_cast<uint32_t>(q) >= span) p0 = 0.f;
              if (static_cast<uint32_t>(q + 1) >= span) p1 = 0.f;
            }
            ppk[16 * c + x / 2] = pack2<BF16>(p0, p1);
          }
        }
        if (c == 1) {
          uint32_t out[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) out[e] = ppk[e];
          tmem_st16(t_row + 64 * h, out);
#pragma unroll
          for (int e = 0; e < 16; ++e) out[e] = ppk[16 + e];
          tmem_st16(t_row + 64 * h + 16, out);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
      // dS pass: dS^T = P^T * dP'^T, packed 16-bit, over dP^T in tensor
      // memory in the column layout of P^T (queries 2i, 2i + 1 of chunk c in
      // column 64h + 16c + i, each chunk landing in columns already read):
      // the A operand of dK.  DQ: also into the 128-byte-swizzled shared
      // tile (row r, 64 queries per 16 KB chunk), the operand of dQ.
      if (!__all_sync(0xffffffffu, mbar_wait(dp_full, it & 1, abort_flag))) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pr[32];
        tmem_ld32(t_row + kColDP + 64 * h + 32 * c, pr);
        uint32_t dsk[16];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const int x = 16 * g + e;
            const float2 d = mul2(unpack2<BF16>(ppk[16 * c + x / 2]),
                                  make_float2(__uint_as_float(pr[x]), __uint_as_float(pr[x + 1])));
            dsk[8 * g + e / 2] = pack2<BF16>(d.x, d.y);
          }
          if constexpr (DQ) {
#pragma unroll
            for (int v = 0; v < 2; ++v) {
              const int unit = (4 * c + 2 * g + v) ^ (r & 7);
              *reinterpret_cast<uint4*>(ds_row + unit * 16) =
                  make_uint4(dsk[8 * g + 4 * v], dsk[8 * g + 4 * v + 1], dsk[8 * g + 4 * v + 2], dsk[8 * g + 4 * v + 3]);
            }
          }
        }
        tmem_st16(t_row + kColDP + 64 * h + 16 * c, dsk);
      }
      tmem_st_wait();
      tc_fence_before();
      if constexpr (DQ) fence_proxy_async_smem();
      mbar_arrive(ds_full);
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ dQ drain, dK/dV epilogue
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // TMEM lane: head-dim index (dQ^T) or query row (dQ)
    const uint32_t t_row = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    bool ok = true;
    for (int it = 0; DQ && it < n_it; ++it) {
      ok = __all_sync(0xffffffffu, mbar_wait(dq_full, it & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const size_t qrow0 = qslab + static_cast<size_t>(i0 + it) * kBwdTile;
      if constexpr (kDqT) {
        // Thread = head-dim index d; a warp's reduction covers 32 consecutive
        // d of one query row (128 contiguous bytes).
        // All 128 columns are read before the columns are released, so the
        // next dP^T product does not wait for the reductions.  Query rows
        // past the sequence in a ragged tile hold exact zeros (masked P) and are
        // reduced like the others; the host pads the accumulator for them.
        float* base = dqacc + qrow0 * D + row;
        uint32_t va[32], vb[32], vc[32], vd[32];
        tmem_ld32(t_row + kColDQ, va);
        tmem_ld32(t_row + kColDQ + 32, vb);
        tmem_ld32(t_row + kColDQ + 64, vc);
        tmem_ld32(t_row + kColDQ + 96, vd);
        tc_fence_before();
        mbar_arrive(dq_free);
#pragma unroll
        for (int q = 0; q < 32; ++q)
          atomicAdd(base + static_cast<size_t>(q) * D, __uint_as_float(va[q]) * scale);
#pragma unroll
        for (int q = 0; q < 32; ++q)
          atomicAdd(base + static_cast<size_t>(32 + q) * D, __uint_as_float(vb[q]) * scale);
#pragma unroll
        for (int q = 0; q < 32; ++q)
          atomicAdd(base + static_cast<size_t>(64 + q) * D, __uint_as_float(vc[q]) * scale);
#pragma unroll
        for (int q = 0; q < 32; ++q)
          atomicAdd(base + static_cast<size_t>(96 + q) * D, __uint_as_float(vd[q]) * scale);
      } else {
        // Thread = query row; 64 head-dim values as 16-byte vector reductions.
        uint32_t va[32], vb[32];
        tmem_ld32(t_row + kColDQ, va);
        tmem_ld32(t_row + kColDQ + 32, vb);
        tc_fence_before();
        mbar_arrive(dq_free);
        float* dst = dqacc + (qrow0 + row) * D;
#pragma unroll
        for (int v = 0; v < 8; ++v)
          atomicAdd(reinterpret_cast<float4*>(dst + 4 * v),
                    make_float4(__uint_as_float(va[4 * v]) * scale, __uint_as_float(va[4 * v + 1]) * scale,
                                __uint_as_float(va[4 * v + 2]) * scale, __uint_as_float(va[4 * v + 3]) * scale));
#pragma unroll
        for (int v = 0; v < 8; ++v)
          atomicAdd(reinterpret_cast<float4*>(dst + 32 + 4 * v),
                    make_float4(__uint_as_float(vb[4 * v]) * scale, __uint_as_float(vb[4 * v + 1]) * scale,
                                __uint_as_float(vb[4 * v + 2]) * scale, __uint_as_float(vb[4 * v + 3]) * scale));
      }
    }
    if (ok && n_it > 0) {
      if (__all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag))) {
        tc_fence_after();
        // dK / dV: M = keys, so the TMEM lane is the key row.
        const size_t grow = krow0 + row;
        const bool live = row < kv_valid;  // padding rows of a ragged key tile are not stored
        uint4* dvd = reinterpret_cast<uint4*>(dv_ptr + grow * D);
        uint4* dkd = reinterpret_cast<uint4*>(dk_ptr + grow * D);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t rv[32], pk[16];
          tmem_ld32(t_row + kColDV + c * 32, rv);
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack2<BF16>(__uint_as_float(rv[2 * e]), __uint_as_float(rv[2 * e + 1]));
          if (live) {
#pragma unroll
            for (int v = 0; v < 4; ++v) dvd[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
          tmem_ld32(t_row + kColDK + c * 32, rv);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack2<BF16>(__uint_as_float(rv[2 * e]) * scale, __uint_as_float(rv[2 * e + 1]) * scale);
          if (live) {
#pragma unroll
            for (int v = 0; v < 4; ++v) dkd[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn
