// bwd_kv_wide_kernel.cuh -- dK and dV of the attention backward at head
// dimension 256, one 64-key tile per CTA.
//
// The backward pass recomputes the probabilities from Q, K and the saved row
// log-sum-exp (page "FlashAttention 核心原理", part 2 item 3).  For a key tile
// K_j, V_j (64 keys) and every query tile Q_i, dO_i (128 rows) that sees it:
//   S  = Q_i K_j^T,  P = exp2(scale log2(e) S - log2(e) LSE_i)
//   dP = dO_i V_j^T, dS = P * (dP - D_i)
//   dV_j^T += dO_i^T P,   dK_j^T += Q_i^T dS
// and at the end dV_j and dK_j = scale * dK_j are written.  dQ comes from
// bwd_dq_kernel (one CTA per query tile, no atomics), so the d = 256
// backward is reproducible bit for bit.
//
// Why this shape: at d = 256 the accumulators of a 128-key tile (dK and dV,
// 128 x 256 fp32 each) would fill all 512 tensor-memory columns, leaving
// none for S and dP.  Keeping them transposed for 64 keys, dV^T and dK^T as
// two 128-row halves of the head dimension each, takes 256 columns, and
// every product keeps a 128-row (M = 128) tensor-core shape:
//   S, dP          M = 128 queries, N = 64 keys,  K = 256 (head dim)
//   dV^T, dK^T     M = 128 head-dim rows (x2), N = 64 keys, K = 128 queries
// All four read both operands from shared memory: Q_i and dO_i are the
// K-major A of S and dP and the MN-major A of dK^T and dV^T; P and dS go
// from the softmax warps to shared memory as the MN-major B operands.
// Shared memory holds one Q_i and one dO_i (64 KB each), so the next query
// tile's Q is loaded once dK^T has read this one, and its dO once dV^T has.
// The next S product, which starts the next tile's softmax, waits for that Q
// load; so per query tile the issue order is S, dP, dK^T, dV^T: dK^T, the
// last reader of Q_i, goes first once dS is written (P is ready earlier, but
// dV^T can wait), and dV^T then runs while Q_{i+1} is in flight.
//
// CTA layout (384 threads, one CTA per SM):
//   warp 0       TMA producer: K_j and V_j once; dO_i, Q_i per query tile
//   warp 1       MMA issuer (one elected lane per group)
//   warp 2       tensor-memory allocation / release
//   warp 3       idle
//   warps 4-7    P and dS for keys [0, 32) of the tile   (thread = query row
//   warps 8-11   P and dS for keys [32, 64)               = TMEM lane)
//                then the epilogue: warpgroup h writes head-dim half h
// Tensor memory (512 columns allocated, 384 used):
//   [0, 64)      S (fp32)
//   [64, 128)    dP (fp32)
//   [128, 256)   dV^T: head-dim half h in columns 128 + 64h + key
//   [256, 384)   dK^T, the same way
#pragma once

#include "sm100.cuh"
#include "tile_order.h"

namespace attn {

struct BwdKvWideLayout {
  static constexpr int D = 256;
  static constexpr int kKeyRows = 64;                    // keys of the CTA
  static constexpr int kQRows = 128;                     // query rows of one step
  static constexpr int kChunks = D * 2 / 128;            // 128-byte column chunks per row
  static constexpr int kKeyChunkBytes = kKeyRows * 128;  // 8 KB
  static constexpr int kQChunkBytes = kQRows * 128;      // 16 KB
  static constexpr int kKeyTileBytes = kKeyRows * D * 2;  // 32 KB
  static constexpr int kQTileBytes = kQRows * D * 2;      // 64 KB
  static constexpr int kPBytes = kQRows * kKeyRows * 2;   // 16 KB: [128 queries][64 keys] 16-bit
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKOff + kKeyTileBytes;
  static constexpr int kQOff = kVOff + kKeyTileBytes;
  static constexpr int kDOOff = kQOff + kQTileBytes;
  static constexpr int kPOff = kDOOff + kQTileBytes;
  static constexpr int kDSOff = kPOff + kPBytes;
  static constexpr int kBarOff = kDSOff + kPBytes;
  // kv_full, q_full, do_full, q_free, do_free, s_full, s_read, dp_full,
  // dp_read, p_full, p_free, ds_full, ds_free, acc_done, mma_done
  static constexpr int kNumBars = 15;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024 <= 232448 ? kBytes + 1024 : 232448;
  static_assert(kBytes <= 232448, "shared memory budget");
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColDP = 64;
  static constexpr uint32_t kColDV = 128;
  static constexpr uint32_t kColDK = 256;
};

// dvec and nlse2 hold D_i and -log2(e) LSE_i per query row of the tensor
// maps' slabs (bwd_pre_kernel).  tm_k and tm_v read 64-row boxes, tm_q and
// tm_do 128-row boxes.  The grid is the 64-key tiles of every problem
// (grid_tiles per problem) in the grouped launch order of tile_order.h;
// causal grids put the first key tiles, which the most query tiles see,
// first.
template <bool BF16, bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    bwd_kv_wide_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const float* __restrict__ dvec, const float* __restrict__ nlse2,
                       uint16_t* __restrict__ dk_ptr, uint16_t* __restrict__ dv_ptr, const int* __restrict__ cu_q,
                       const int* __restrict__ cu_k, int H, int Nq, int Nk, int bottom_right, float scale,
                       float scale_log2, int problems, int grid_tiles, int group) {
  using L = BwdKvWideLayout;
  constexpr int D = L::D;
  constexpr int kKR = L::kKeyRows;
  constexpr int kQR = L::kQRows;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;
  uint64_t* do_full = bars + 2;
  uint64_t* q_free = bars + 3;    // dK^T(i) has read Q_i
  uint64_t* do_free = bars + 4;   // dV^T(i) has read dO_i
  uint64_t* s_full = bars + 5;
  uint64_t* s_read = bars + 6;    // 256 arrivals: S loaded by the softmax warps
  uint64_t* dp_full = bars + 7;
  uint64_t* dp_read = bars + 8;   // 256 arrivals
  uint64_t* p_full = bars + 9;    // 256 arrivals: P written to shared memory
  uint64_t* p_free = bars + 10;   // dV^T has read P
  uint64_t* ds_full = bars + 11;  // 256 arrivals
  uint64_t* ds_free = bars + 12;  // dK^T has read dS
  uint64_t* acc_done = bars + 13;
  uint64_t* mma_done = bars + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // The problem of this CTA (as in the forward): slab z, rows [q0, q0 + nq)
  // of the queries and [k0, k0 + nk) of the keys, offsets of a packed batch
  // clamped to the slab.
  int px, kt;
  grouped_order(blockIdx.x, problems, grid_tiles, group, &px, &kt);
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
  }
  const int nkt = (nk + kKR - 1) / kKR;
  if (kt >= nkt) return;  // a sequence shorter than the grid
  const int key0 = kt * kKR;                                // first key of the tile
  const int keys = nk - key0 < kKR ? nk - key0 : kKR;       // valid keys of the tile
  const int off = bottom_right ? nk - nq : 0;
  // Query tiles that see the tile: all of them, or (causal: query r sees key
  // k iff k <= r + off) those from the one holding row key0 - off on.
  const int nqt = (nq + kQR - 1) / kQR;
  int i0 = 0;
  if (CAUSAL) {
    const int first_row = key0 - off;
    i0 = first_row <= 0 ? 0 : first_row / kQR;
  }
  const int n_it = nqt > i0 ? nqt - i0 : 0;
  const size_t krow0 = static_cast<size_t>(z) * Nk + k0 + key0;  // first key row of the tile
  if (n_it == 0) {
    // No query sees these keys: dK = dV = 0.
    for (int e = threadIdx.x; e < keys * D / 8; e += blockDim.x) {
      reinterpret_cast<uint4*>(dk_ptr + krow0 * D)[e] = make_uint4(0u, 0u, 0u, 0u);
      reinterpret_cast<uint4*>(dv_ptr + krow0 * D)[e] = make_uint4(0u, 0u, 0u, 0u);
    }
    return;
  }

  // Refuse to run (and report) if alignment left too little shared memory.
  if (static_cast<uint32_t>(smem - smem_raw) + L::kBytes > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) atomicExch(&g_device_status, kStatusSmem);
    return;
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);  // kv_full .. s_full
    mbar_init(s_read, 256);
    mbar_init(dp_full, 1);
    mbar_init(dp_read, 256);
    mbar_init(p_full, 256);
    mbar_init(p_free, 1);
    mbar_init(ds_full, 256);
    mbar_init(ds_free, 1);
    mbar_init(acc_done, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
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
      mbar_arrive_expect_tx(kv_full, 2 * L::kKeyTileBytes);
      for (int c = 0; c < L::kChunks; ++c) {
        tma_load_3d(smem + L::kKOff + c * L::kKeyChunkBytes, &tm_k, kv_full, c * 64, k0 + key0, z);
        tma_load_3d(smem + L::kVOff + c * L::kKeyChunkBytes, &tm_v, kv_full, c * 64, k0 + key0, z);
      }
      int n_do = 0, n_q = 0;  // loads issued
      bool ok = true;
      for (int it = 0; it < n_it; ++it) {
        const int row0 = q0 + (i0 + it) * kQR;
        if (it > 0 && !(ok = mbar_wait(q_free, (it - 1) & 1, abort_flag))) break;
        mbar_arrive_expect_tx(q_full, L::kQTileBytes);
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(smem + L::kQOff + c * L::kQChunkBytes, &tm_q, q_full, c * 64, row0, z);
        ++n_q;
        if (it > 0 && !(ok = mbar_wait(do_free, (it - 1) & 1, abort_flag))) break;
        mbar_arrive_expect_tx(do_full, L::kQTileBytes);
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(smem + L::kDOOff + c * L::kQChunkBytes, &tm_do, do_full, c * 64, row0, z);
        ++n_do;
      }
      if (!ok) {
        // Let the copies already issued land before the CTA exits.
        mbar_drain(kv_full, 0);
        if (n_do > 0) mbar_drain(do_full, (n_do - 1) & 1);
        if (n_q > 0) mbar_drain(q_full, (n_q - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdS = idesc_f16(BF16, 128, kKR, false, false);  // K-major x K-major
    constexpr uint32_t kIdT = idesc_f16(BF16, 128, kKR, true, true);    // MN-major x MN-major
    const uint32_t base = smem_u32(smem);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    // K-major SW128: 32 bytes per K step of 16 inside a 128-byte row, one
    // chunk per 64 head-dim columns (16 KB for 128 query rows, 8 KB for 64
    // keys).
    auto kstep_q = [](int ks) { return static_cast<uint64_t>(((ks >> 2) * L::kQChunkBytes + (ks & 3) * 32) >> 4); };
    auto kstep_k = [](int ks) { return static_cast<uint64_t>(((ks >> 2) * L::kKeyChunkBytes + (ks & 3) * 32) >> 4); };
    // S or dP = X K^T with X = Q_i or dO_i (A) and Y = K_j or V_j (B).
    auto issue_qk = [&](uint32_t d_col, uint32_t a_off, uint32_t b_off) {
      const uint64_t ad = sdesc_sw128(base + a_off, 16, 1024);
      const uint64_t bd = sdesc_sw128(base + b_off, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        mma_ss(tmem + d_col, ad + kstep_q(ks), bd + kstep_k(ks), kIdS, ks > 0 ? 1u : 0u);
    };
    // Acc^T += X^T Y for head-dim halves hh: A = X^T MN-major (chunks 2hh and
    // 2hh+1 of X, 16 KB apart; 16 query rows of 128 bytes per K step), B =
    // Y [128 queries][64 keys] MN-major (one 128-byte chunk).
    auto issue_acc = [&](uint32_t d_col, uint32_t a_off, uint32_t b_off, bool first) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint64_t ad = sdesc_sw128(base + a_off + 2 * hh * L::kQChunkBytes, L::kQChunkBytes, 1024);
        const uint64_t bd = sdesc_sw128(base + b_off, L::kQChunkBytes, 1024);
#pragma unroll
        for (int ks = 0; ks < kQR / 16; ++ks)
          mma_ss(tmem + d_col + 64 * hh, ad + 128 * ks, bd + 128 * ks, kIdT, (!first || ks > 0) ? 1u : 0u);
      }
    };
    bool ok = wait_all(kv_full, 0);
    for (int it = 0; ok && it < n_it; ++it) {
      const uint32_t par = it & 1, prev = (it - 1) & 1;
      // S(it) = Q_i K_j^T.
      if (!(ok = wait_all(q_full, par))) break;
      if (it > 0 && !(ok = wait_all(s_read, prev))) break;
      tc_fence_after();
      if (elect_one()) {
        issue_qk(L::kColS, L::kQOff, L::kKOff);
        mma_commit(s_full);
      }
      __syncwarp();
      // dP(it) = dO_i V_j^T over dP(it-1), which the softmax warps have loaded.
      if (!(ok = wait_all(do_full, par))) break;
      if (it > 0 && !(ok = wait_all(dp_read, prev))) break;
      tc_fence_after();
      if (elect_one()) {
        issue_qk(L::kColDP, L::kDOOff, L::kVOff);
        mma_commit(dp_full);
      }
      __syncwarp();
      // dK^T += Q_i^T dS(it): then Q_i and dS are free.
      if (!(ok = wait_all(ds_full, par))) break;
      tc_fence_after();
      if (elect_one()) {
        issue_acc(L::kColDK, L::kQOff, L::kDSOff, it == 0);
        mma_commit(ds_free);
        mma_commit(q_free);
      }
      __syncwarp();
      // dV^T += dO_i^T P(it): then dO_i and P are free.
      if (!(ok = wait_all(p_full, par))) break;
      tc_fence_after();
      if (elect_one()) {
        issue_acc(L::kColDV, L::kDOOff, L::kPOff, it == 0);
        mma_commit(p_free);
        mma_commit(do_free);
        if (it == n_it - 1) mma_commit(acc_done);
      }
      __syncwarp();
    }
    if (elect_one()) mma_commit(mma_done);
    __syncwarp();
    mbar_drain(mma_done, 0);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ P, dS, epilogue
    const int h = (warp - 4) >> 2;   // keys [32h, 32h + 32) of the tile
    const int wq = warp & 3;         // 32-lane TMEM slice of this warp
    const int row = wq * 32 + lane;  // query row within a query tile
    const uint32_t t_row = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float2 c2 = make_float2(scale_log2, scale_log2);
    // P and dS rows in shared memory: [128 queries][64 keys] 16-bit, 128-byte
    // swizzled; this thread writes 16-byte units 4h .. 4h+3 of its row.
    uint8_t* p_row = smem + L::kPOff + row * 128;
    uint8_t* ds_row = smem + L::kDSOff + row * 128;
    auto store_row = [&](uint8_t* dst, const uint32_t (&pk)[16]) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<uint4*>(dst + (((4 * h + u) ^ (row & 7)) * 16)) =
            make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
    };
    bool ok = true;
    for (int it = 0; ok && it < n_it; ++it) {
      const uint32_t par = it & 1, prev = (it - 1) & 1;
      const int qrow = (i0 + it) * kQR + row;  // query row in the sequence
      const bool live = qrow < nq;              // padding rows of a ragged tile: P = dS = 0
      const size_t grow = static_cast<size_t>(z) * Nq + q0 + qrow;
      const float nl = live ? nlse2[grow] : 0.f;
      const float dr = live ? dvec[grow] : 0.f;
      // Keys of this warpgroup kept for this row: column c iff c <= lim.
      int lim = -1;
      if (live) {
        int last = nk - 1;
        if (CAUSAL && qrow + off < last) last = qrow + off;
        lim = last - (key0 + 32 * h);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, par, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float p[32];
      {
        uint32_t r[32];
        tmem_ld32(t_row + L::kColS + 32 * h, r);
        tc_fence_before();
        mbar_arrive(s_read);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 a = fma2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), c2,
                                make_float2(nl, nl));
          p[2 * i] = ex2(a.x);
          p[2 * i + 1] = ex2(a.y);
        }
      }
      if (__any_sync(0xffffffffu, lim < 31)) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (c > lim) p[c] = 0.f;
      }
      {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack2<BF16>(p[2 * i], p[2 * i + 1]);
        // dV^T(it-1) has read the previous P.
        if (it > 0) ok = __all_sync(0xffffffffu, mbar_wait(p_free, prev, abort_flag));
        if (!ok) break;
        store_row(p_row, pk);
        fence_proxy_async_smem();
        mbar_arrive(p_full);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(dp_full, par, abort_flag));
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t r[32];
        tmem_ld32(t_row + L::kColDP + 32 * h, r);
        tc_fence_before();
        mbar_arrive(dp_read);
        const float2 nd2 = make_float2(-dr, -dr);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 dpm = add2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), nd2);
          const float2 ds = mul2(make_float2(p[2 * i], p[2 * i + 1]), dpm);
          pk[i] = pack2<BF16>(ds.x, ds.y);
        }
        // dK^T(it-1) has read the previous dS.
        if (it > 0) ok = __all_sync(0xffffffffu, mbar_wait(ds_free, prev, abort_flag));
        if (!ok) break;
        store_row(ds_row, pk);
        fence_proxy_async_smem();
        mbar_arrive(ds_full);
      }
    }
    // Epilogue: warpgroup h holds head-dim half h of dV^T and dK^T (TMEM lane
    // = head-dim index 128h + row, column = key); each thread writes its
    // head-dim column of the tile's valid keys (a warp covers 64 contiguous
    // bytes of a key row per store).
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(acc_done, 0, abort_flag));
    if (ok) {
      tc_fence_after();
      const int dd = 128 * h + row;
#pragma unroll 1
      for (int t = 0; t < 2; ++t) {
        uint16_t* dst = (t == 0 ? dv_ptr : dk_ptr) + krow0 * D + dd;
        const float mult = t == 0 ? 1.f : scale;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          tmem_ld32(t_row + (t == 0 ? L::kColDV : L::kColDK) + 64 * h + 32 * c, r);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const uint32_t pr = pack2<BF16>(__uint_as_float(r[i]) * mult, __uint_as_float(r[i + 1]) * mult);
            const int key = 32 * c + i;
            if (key < keys) dst[static_cast<size_t>(key) * D] = static_cast<uint16_t>(pr & 0xFFFFu);
            if (key + 1 < keys) dst[static_cast<size_t>(key + 1) * D] = static_cast<uint16_t>(pr >> 16);
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
