// bwd_dq_kernel.cuh -- dQ of the attention backward, one query tile per CTA.
//
// The backward pass recomputes the attention probabilities from Q, K and the
// saved row log-sum-exp instead of storing them (page "FlashAttention 核心原理",
// part 2 item 3).  bwd_main_kernel does so per key tile and accumulates dK and
// dV; this kernel does so per query tile and accumulates
//   dQ_i = scale * sum_j dS_ij K_j,   dS = P * (dO V^T - D),
//   P = exp(scale * Q K^T - LSE)
// over the key tiles j that the query tile sees.  Each CTA owns its dQ rows,
// so dQ needs no atomic additions and comes out the same, bit for bit, on
// every run; together with bwd_main_kernel<..., DQ = false> it is the
// reproducible backward.
//
// CTA layout (384 threads, one CTA per SM):
//   warp 0       TMA producer: Q_i and dO_i once, then K_0, V_0, K_1, V_1, ...
//                through a ring of shared-memory slots
//   warp 1       MMA issuer (one elected lane per group)
//   warp 2       tensor-memory allocation / release
//   warp 3       idle
//   warps 4-7    P and dS for key columns [0, 64) of every key tile
//   warps 8-11   P and dS for key columns [64, 128)
//                (thread = query row = TMEM lane: a row's LSE and D are
//                per-thread values; at the start each warpgroup copies half
//                of the head dimension of Q and dO into tensor memory, and at
//                the end writes half of the head dimension of dQ)
// Tensor memory (512 columns at d = 128):
//   [0, 128)        S (fp32)
//   [128, 256)      dP = dO V^T (fp32); dS of the tile is written over it,
//                   16-bit packed, keys [64h, 64h+64) in columns
//                   128 + [64h, 64h+32)
//   [256, 256+D)    dQ accumulator (fp32)
//   then Q and dO, 16-bit pairs (D/2 columns each): the A operands of S and dP
// Products per key tile j: S(j) = Q K_j^T and dP(j) = dO V_j^T with A from
// tensor memory (only K_j or V_j is read from shared memory), and
// dQ += dS(j) K_j with dS from tensor memory.  Issue order: S(0), dP(0), then
// per j: S(j+1) as soon as the softmax warps have loaded S(j) into
// registers, dQ(j) once they have written dS(j), dP(j+1) behind dQ(j) (which
// reads the dS it overwrites).  The warps find S(j+1) ready when they finish
// tile j and wait for dP(j+1) only while dQ(j) and dP(j+1) run.
// d = 256 (the only dQ kernel of the d = 256 backward): key tiles of 64 rows
// (each warpgroup owns 32 key columns), S in [0, 64), dP in [64, 128), the
// dQ accumulator in [128, 384) and Q in [384, 512); dO has no room in tensor
// memory and stays in shared memory, so dP reads both operands from there.
// Once Q is in tensor memory its staging area holds two more ring slots.
#pragma once

#include "sm100.cuh"
#include "tile_order.h"

namespace attn {

template <int D>
struct BwdDqLayout {
  static constexpr int kTileRows = 128;                 // query rows of a CTA
  static constexpr int kKeyRows = D == 256 ? 64 : 128;  // keys of a key tile
  static constexpr int kKeyHalf = kKeyRows / 2;         // keys of one softmax warpgroup
  static constexpr int kRowBytes = D * 2;
  static constexpr int kChunks = kRowBytes / 128;        // 128-byte column chunks per row
  static constexpr int kChunkBytes = kTileRows * 128;    // one chunk of Q or dO
  static constexpr int kKeyChunkBytes = kKeyRows * 128;  // one chunk of K or V
  static constexpr int kTileBytes = kTileRows * kRowBytes;
  static constexpr int kKeyTileBytes = kKeyRows * kRowBytes;
  // d = 256: dO stays in shared memory (the A operand of dP has no room in
  // tensor memory), and once Q has been copied into tensor memory its
  // staging area serves as two more ring slots.
  static constexpr bool kWide = D == 256;
  static constexpr int kSlots = D == 64 ? 10 : 5;       // K/V ring slots
  static constexpr int kOwnSlots = kWide ? 3 : kSlots;  // slots after dO; the rest alias Q
  static constexpr int kQOff = 0;
  static constexpr int kDOOff = kQOff + kTileBytes;
  static constexpr int kRingOff = kDOOff + kTileBytes;
  static constexpr int kBarOff = kRingOff + kOwnSlots * kKeyTileBytes;
  static_assert(kWide ? (kSlots - kOwnSlots) * kKeyTileBytes <= kTileBytes : kOwnSlots == kSlots, "ring");
  // qd_full, kv_full[kSlots], kv_empty[kSlots], s_full, s_read, dp_full,
  // ds_full, dq_done, mma_done, qd_tmem
  static constexpr int kNumBars = 1 + 2 * kSlots + 7;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024 <= 232448 ? kBytes + 1024 : 232448;
  static_assert(kBytes <= 232448, "shared memory budget");
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColDP = kKeyRows;
  static constexpr uint32_t kColDQ = 2 * kKeyRows;
  static constexpr uint32_t kColQ = kColDQ + D;      // Q, 16-bit pairs
  static constexpr uint32_t kColDO = kColQ + D / 2;  // dO, 16-bit pairs (not at d = 256)
  static_assert((kWide ? kColQ : kColDO) + D / 2 <= 512, "tensor memory budget");
};

// dvec and nlse2 hold D_i and -log2(e) LSE_i per query row of the tensor
// maps' slabs (bwd_pre_kernel); dq_ptr is the 16-bit dQ.  The grid is the
// query tiles of every problem in the grouped launch order of tile_order.h.
template <int D, bool BF16, bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const float* __restrict__ dvec, const float* __restrict__ nlse2, uint16_t* __restrict__ dq_ptr,
                  const int* __restrict__ cu_q, const int* __restrict__ cu_k, int H, int Nq, int Nk,
                  int bottom_right, float scale, float scale_log2, int problems, int grid_tiles, int group) {
  using L = BwdDqLayout<D>;
  constexpr int kT = L::kTileRows;
  constexpr int kKR = L::kKeyRows;
  constexpr int kKW = L::kKeyHalf;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* qd_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + L::kSlots;
  uint64_t* s_full = kv_empty + L::kSlots;
  uint64_t* s_read = s_full + 1;            // 256 arrivals: S loaded by the softmax warps
  uint64_t* dp_full = s_read + 1;
  uint64_t* ds_full = dp_full + 1;          // 256 arrivals: dS written
  uint64_t* dq_done = ds_full + 1;
  uint64_t* mma_done = dq_done + 1;
  uint64_t* qd_tmem = mma_done + 1;         // 256 arrivals: Q and dO copied into tensor memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // The problem of this CTA (as in the forward): slab z, rows [q0, q0 + nq)
  // of the queries and [k0, k0 + nk) of the keys, offsets of a packed batch
  // clamped to the slab.
  int px, ty;
  grouped_order(blockIdx.x, problems, grid_tiles, group, &px, &ty);
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
  const int nqt = (nq + kT - 1) / kT;
  const int nkt = (nk + kKR - 1) / kKR;
  if (ty >= nqt) return;  // a sequence shorter than the grid
  // Causal: the heaviest query tiles are launched first.
  const int qt = CAUSAL ? (nqt - 1 - ty) : ty;
  // Key tiles this query tile sees (causal: query i sees key k iff
  // k <= i + off, off = 0 top-left, nk - nq bottom-right).
  const int off = bottom_right ? nk - nq : 0;
  int n = nkt;
  if (CAUSAL) {
    const int last_row = qt * kT + kT - 1 < nq - 1 ? qt * kT + kT - 1 : nq - 1;
    const int last_key = last_row + off < nk - 1 ? last_row + off : nk - 1;
    n = last_key < 0 ? 0 : last_key / kKR + 1;
  }
  const size_t grow0 = static_cast<size_t>(z) * Nq + q0 + static_cast<size_t>(qt) * kT;  // first row of the tile
  if (n == 0) {
    // No row of this tile sees a key: its softmax is empty and dQ = 0.
    const int rows = nq - qt * kT < kT ? nq - qt * kT : kT;
    for (int e = threadIdx.x; e < rows * D / 8; e += blockDim.x)
      reinterpret_cast<uint4*>(dq_ptr + grow0 * D)[e] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }

  // Refuse to run (and report) if alignment left too little shared memory.
  if (static_cast<uint32_t>(smem - smem_raw) + L::kBytes > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) atomicExch(&g_device_status, kStatusSmem);
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    for (int i = 0; i < L::kSlots; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_read, 256);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 256);
    mbar_init(dq_done, 1);
    mbar_init(mma_done, 1);
    mbar_init(qd_tmem, 256);
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

  // Ring items: K_j is item 2j, V_j item 2j + 1 (j < n).
  auto ring_off = [](int slot) {
    return slot < L::kOwnSlots ? L::kRingOff + slot * L::kKeyTileBytes
                               : L::kQOff + (slot - L::kOwnSlots) * L::kKeyTileBytes;
  };
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(qd_full, 2 * L::kTileBytes);
      for (int c = 0; c < L::kChunks; ++c) {
        tma_load_3d(smem + L::kQOff + c * L::kChunkBytes, &tm_q, qd_full, c * 64, q0 + qt * kT, z);
        tma_load_3d(smem + L::kDOOff + c * L::kChunkBytes, &tm_do, qd_full, c * 64, q0 + qt * kT, z);
      }
      int item = 0;
      bool ok = true;
      for (; ok && item < 2 * n; ++item) {
        const int slot = item % L::kSlots;
        // d = 256: the slots in the Q staging area are free once Q is in
        // tensor memory.
        if (L::kWide && item == L::kOwnSlots && !mbar_wait(qd_tmem, 0, abort_flag)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&kv_empty[slot], ((item / L::kSlots) & 1) ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&kv_full[slot], L::kKeyTileBytes);
        uint8_t* dst = smem + ring_off(slot);
        const CUtensorMap* map = (item & 1) ? &tm_v : &tm_k;
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(dst + c * L::kKeyChunkBytes, map, &kv_full[slot], c * 64, k0 + (item >> 1) * kKR, z);
      }
      if (!ok) {
        // Let the copies already issued land before the CTA exits.
        mbar_drain(qd_full, 0);
        const int first = item > L::kSlots ? item - L::kSlots : 0;
        for (int i = first; i < item; ++i) mbar_drain(&kv_full[i % L::kSlots], (i / L::kSlots) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdS = idesc_f16(BF16, 128, kKR, false, false);  // A (TMEM or K-major) x K-major
    constexpr uint32_t kIdQ = idesc_f16(BF16, 128, D, false, true);     // dS (TMEM) x K MN-major
    const uint32_t smem_base = smem_u32(smem);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    auto slot_addr = [&](int item) { return smem_base + ring_off(item % L::kSlots); };
    auto wait_item = [&](int item) { return wait_all(&kv_full[item % L::kSlots], (item / L::kSlots) & 1); };
    // K-major SW128 operands: 32 bytes per K step of 16 inside a 128-byte
    // row, one chunk per 64 columns (kChunkBytes for the 128-row Q and dO,
    // kKeyChunkBytes for K and V); A from tensor memory: 8 columns per step.
    auto kstep_q = [](int ks) { return static_cast<uint64_t>(((ks >> 2) * L::kChunkBytes + (ks & 3) * 32) >> 4); };
    auto kstep_k = [](int ks) { return static_cast<uint64_t>(((ks >> 2) * L::kKeyChunkBytes + (ks & 3) * 32) >> 4); };
    auto issue_s = [&](int j) {  // S(j) = Q K_j^T
      const uint64_t kd = sdesc_sw128(slot_addr(2 * j), 16, 1024);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        mma_ts(tmem + L::kColS, tmem + L::kColQ + 8 * ks, kd + kstep_k(ks), kIdS, ks > 0 ? 1u : 0u);
    };
    auto issue_dp = [&](int j) {  // dP(j) = dO V_j^T (d = 256: dO from shared memory)
      const uint64_t vd = sdesc_sw128(slot_addr(2 * j + 1), 16, 1024);
      const uint64_t od = sdesc_sw128(smem_base + L::kDOOff, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        if constexpr (L::kWide)
          mma_ss(tmem + L::kColDP, od + kstep_q(ks), vd + kstep_k(ks), kIdS, ks > 0 ? 1u : 0u);
        else
          mma_ts(tmem + L::kColDP, tmem + L::kColDO + 8 * ks, vd + kstep_k(ks), kIdS, ks > 0 ? 1u : 0u);
      }
    };
    // dQ += dS(j) K_j: A = dS over dP (key step ks of 16 keys: the keys
    // [kKW h, kKW h + kKW) of warpgroup h sit in columns kKW h + [0, kKW/2),
    // 8 per step), B = K_j MN-major (16 key rows of 128 bytes per step).
    auto issue_dq = [&](int j) {
      const uint64_t kmn = sdesc_sw128(slot_addr(2 * j), L::kKeyChunkBytes, 1024);
      constexpr int kStepsPerHalf = kKW / 16;
#pragma unroll
      for (int ks = 0; ks < kKR / 16; ++ks) {
        const uint32_t ds_col = tmem + L::kColDP + kKW * (ks / kStepsPerHalf) + 8 * (ks % kStepsPerHalf);
        mma_ts(tmem + L::kColDQ, ds_col, kmn + 128 * ks, kIdQ, (j > 0 || ks > 0) ? 1u : 0u);
      }
    };
    bool ok = wait_all(qd_tmem, 0) && wait_item(0) && wait_item(1);
    if (ok) {
      tc_fence_after();
      if (elect_one()) {
        issue_s(0);
        mma_commit(s_full);
        issue_dp(0);
        mma_commit(dp_full);
        mma_commit(&kv_empty[1 % L::kSlots]);  // V_0 read
      }
      __syncwarp();
    }
    for (int j = 0; ok && j < n; ++j) {
      if (j + 1 < n) {
        // S(j+1) overwrites S(j): the softmax warps have loaded it.
        if (!(ok = wait_all(s_read, j & 1))) break;
        if (!(ok = wait_item(2 * j + 2))) break;
        tc_fence_after();
        if (elect_one()) {
          issue_s(j + 1);
          mma_commit(s_full);
        }
        __syncwarp();
      }
      if (!(ok = wait_all(ds_full, j & 1))) break;
      if (j + 1 < n && !(ok = wait_item(2 * j + 3))) break;
      tc_fence_after();
      if (elect_one()) {
        issue_dq(j);
        mma_commit(&kv_empty[(2 * j) % L::kSlots]);  // K_j read by S(j) and dQ(j)
        if (j == n - 1) mma_commit(dq_done);
        if (j + 1 < n) {
          issue_dp(j + 1);  // over dS(j), which dQ(j) (issued above) reads first
          mma_commit(dp_full);
          mma_commit(&kv_empty[(2 * j + 3) % L::kSlots]);  // V_{j+1} read
        }
      }
      __syncwarp();
    }
    if (elect_one()) mma_commit(mma_done);
    __syncwarp();
    mbar_drain(mma_done, 0);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ P, dS, dQ epilogue
    const int h = (warp - 4) >> 2;   // key columns [64h, 64h + 64) of every key tile
    const int wq = warp & 3;         // 32-lane TMEM slice of this warp
    const int row = wq * 32 + lane;  // query row within the tile
    const uint32_t t_row = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const bool live = qt * kT + row < nq;  // padding rows of a ragged tile: zero terms, not stored
    const size_t grow = grow0 + row;
    // P = exp2(scale log2(e) q.k - log2(e) LSE); rows that see no key have
    // every key masked (their -log2(e) LSE is stored as 0).
    const float nl = live ? nlse2[grow] : 0.f;
    const float dr = live ? dvec[grow] : 0.f;
    const float2 c2 = make_float2(scale_log2, scale_log2), nl2 = make_float2(nl, nl);
    // Q and dO -> tensor memory: this thread copies its row's half of the
    // head dimension (16-byte units of the 128-byte swizzled tiles) as
    // 32-bit words of two 16-bit values, the lowest index in the low bits.
    bool ok = __all_sync(0xffffffffu, mbar_wait(qd_full, 0, abort_flag));
    if constexpr (L::kWide) {
      // d = 256: Q only; each warpgroup copies two whole chunks of its row.
      if (ok) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint8_t* src = smem + L::kQOff + (2 * h + c) * L::kChunkBytes + row * 128;
          uint32_t w[32];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint4 v4 = *reinterpret_cast<const uint4*>(src + ((u ^ (row & 7)) * 16));
            w[4 * u] = v4.x; w[4 * u + 1] = v4.y; w[4 * u + 2] = v4.z; w[4 * u + 3] = v4.w;
          }
          tmem_st32(t_row + L::kColQ + 64 * h + 32 * c, w);
        }
        tmem_st_wait();
        tc_fence_before();
      }
    } else if (ok) {
      constexpr bool kTwoChunks = L::kRowBytes == 256;  // each warpgroup copies one whole chunk
      constexpr int kUnits = L::kRowBytes / 32;          // 16-byte units in half a row
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const uint8_t* src = smem + (m == 0 ? L::kQOff : L::kDOOff) + (kTwoChunks ? h * L::kChunkBytes : 0) + row * 128;
        uint32_t w[4 * kUnits];
#pragma unroll
        for (int u = 0; u < kUnits; ++u) {
          const int unit = (kTwoChunks ? u : kUnits * h + u) ^ (row & 7);
          const uint4 v4 = *reinterpret_cast<const uint4*>(src + unit * 16);
          w[4 * u] = v4.x; w[4 * u + 1] = v4.y; w[4 * u + 2] = v4.z; w[4 * u + 3] = v4.w;
        }
        const uint32_t col = (m == 0 ? L::kColQ : L::kColDO) + (D / 4) * h;
        if constexpr (kTwoChunks)
          tmem_st32(t_row + col, w);
        else
          tmem_st16(t_row + col, w);
      }
      tmem_st_wait();
      tc_fence_before();
    }
    mbar_arrive(qd_tmem);
    for (int j = 0; ok && j < n; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // Keys past nk (ragged last tile) and, causal, keys after query + off
      // get P = 0: key column c is kept iff c <= lim.
      const int kv_valid = nk - j * kKR;
      const int diag_lim = qt * kT - j * kKR + off;
      const bool masked = (CAUSAL && diag_lim < kKR - 1) || kv_valid < kKR;
      int lim = kv_valid - 1;
      if (CAUSAL && diag_lim + row < lim) lim = diag_lim + row;
      float p[kKW];
#pragma unroll
      for (int c = 0; c < kKW / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(t_row + L::kColS + kKW * h + 32 * c, r);
        if (c == kKW / 32 - 1) {  // S is in registers: S(j+1) may overwrite it
          tc_fence_before();
          mbar_arrive(s_read);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 a = fma2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), c2, nl2);
          p[32 * c + 2 * i] = ex2(a.x);
          p[32 * c + 2 * i + 1] = ex2(a.y);
        }
      }
      if (masked) {
#pragma unroll
        for (int i = 0; i < kKW; ++i)
          if (kKW * h + i > lim) p[i] = 0.f;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(dp_full, j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // dS = P (dP - D), 16-bit, over dP: keys 2i, 2i + 1 of the warpgroup in
      // column kColDP + kKW h + i.  The kKW dP values are loaded first, since
      // the packed dS lands in the first half of the warpgroup's dP columns.
      const float2 nd2 = make_float2(-dr, -dr);
      uint32_t r[kKW];
      if constexpr (kKW == 64)
        tmem_ld64(t_row + L::kColDP + kKW * h, r);
      else
        tmem_ld32(t_row + L::kColDP + kKW * h, r);
#pragma unroll
      for (int c = 0; c < kKW / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 dpm = add2(make_float2(__uint_as_float(r[32 * c + 2 * i]), __uint_as_float(r[32 * c + 2 * i + 1])), nd2);
          const float2 ds = mul2(make_float2(p[32 * c + 2 * i], p[32 * c + 2 * i + 1]), dpm);
          pk[i] = pack2<BF16>(ds.x, ds.y);
        }
        tmem_st16(t_row + L::kColDP + kKW * h + 16 * c, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    // Epilogue: dQ = scale * (the accumulator); this warpgroup writes its
    // half of the head dimension.
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(dq_done, 0, abort_flag));
    if (ok) {
      tc_fence_after();
      uint4* dst = reinterpret_cast<uint4*>(dq_ptr + grow * D + (D / 2) * h);
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t r[32];
        tmem_ld32(t_row + L::kColDQ + (D / 2) * h + 32 * c, r);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack2<BF16>(__uint_as_float(r[2 * i]) * scale, __uint_as_float(r[2 * i + 1]) * scale);
        if (live) {
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
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
