// fwd_kernel.cuh -- fused attention forward for sm_100a.
//
// Computes, for one (batch, head) slice and one 128-row query tile,
//   S = Q K^T (tcgen05 MMA into tensor memory), the online softmax over the
//   key tiles (running row maximum m and row sum l, rescaling with exp2),
//   P cast to 16-bit in tensor memory, O += P V (tcgen05 MMA with P read from
//   tensor memory), and the epilogue O / l and LSE = ln2 * (m + log2 l).
// This is the tiled, fused algorithm of the page "FlashAttention 核心原理"
// (part 2, tiling and kernel fusion) with the online softmax named on the
// page "Flash Attention 落地评估" (section 4); S never leaves the SM.
//
// Both products read their A operand from tensor memory (Q for S = Q K^T,
// P for O += P V) and stream only K or V from shared memory.  A 128x128x16
// MMA with both operands in shared memory reads 8 KB in its 64 cycles, all
// of the SM's shared-memory bandwidth; with A in tensor memory it needs half,
// which leaves room for the TMA writes of the K/V ring.
//
// The grid is persistent: one CTA per SM walks a share of the query tiles
// (unit_at in tile_order.h), so one tile's epilogue overlaps the next tile's
// Q load and first products, and the K/V ring, the S buffers and every
// barrier run on across tiles (their phases count over all of the CTA's key
// tiles).  Short grids lose no time to a CTA's set-up (barriers, tensor
// memory, descriptor prefetch) per tile.
//
// CTA layout (384 threads, one CTA per SM):
//   warp 0       TMA producer: per query tile Q, then K_0, K_1, V_0, K_2,
//                V_1, ... through a ring of shared-memory slots
//   warp 1       MMA issuer (one elected lane per group)
//   warp 2       tensor-memory allocation / release
//   warp 3       set-up: the ones tile and the table of decoded work units
//   warps 4-7    softmax for key columns [0, 64) of every key tile
//   warps 8-11   softmax for key columns [64, 128)
//                (thread = query row = TMEM lane; the two warpgroups
//                exchange their partial row maxima through shared memory,
//                copy each query tile's Q into tensor memory -- the next
//                tile's before this one's epilogue -- and write O through a
//                shared-memory staging tile and TMA stores)
//
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   [0, D/2)     Q, 16-bit pairs (A operand of S = Q K^T)
//   [64, 192)    S buffer 0     [192, 320)  S buffer 1
//                (P of a buffer is packed 16-bit in place: the warpgroup
//                owning key columns [64h, 64h+64) writes their P into
//                buffer columns [64h, 64h+32))
//   [320, 320+D) O
//   [320+D, 336+D) L = P 1: the row sums of the rounded 16-bit P that the
//                O product uses, accumulated (and rescaled) like O, so that
//                O / L is a weighted mean of V rows with weights summing to one
// Issue order: S(0), S(1), then per key tile j: PV(j) and L(j), S(j+2) --
// the softmax of tile j+1 overlaps these products.
#pragma once

#include "sm100.cuh"
#include "tile_order.h"

namespace attn {

constexpr int kTile = 128;  // rows of a query tile and of a key/value tile

// F8: Q, K and V are E4M3 bytes (d = 128 only) instead of 16-bit values.
template <int D, bool F8 = false>
struct FwdLayout {
  static constexpr int kElemBytes = F8 ? 1 : 2;
  static constexpr int kRowBytes = D * kElemBytes;        // one row of Q, K or V
  static constexpr int kChunks = kRowBytes / 128;         // 128-byte column chunks per row (>= 1)
  static constexpr int kChunkElems = 128 / kElemBytes;    // elements of one chunk (TMA box width)
  static constexpr int kChunkBytes = kTile * 128;         // one 128-row chunk
  static constexpr int kTileBytes = kTile * kRowBytes;    // one 128 x D tile
  static constexpr int kKeysPerStep = 32 / kElemBytes;    // keys per MMA K step (32 bytes)
  static constexpr bool kWide = D == 256;                 // see below
  static constexpr int kSlots = kWide ? 2 : (kTileBytes == 32768 ? 4 : 10);  // K/V ring slots
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = kQOff + kTileBytes;
  // d <= 128: the epilogue stages the 16-bit O tile here (128-byte
  // swizzled chunks of 64 columns, the layout of a TMA load) and writes it
  // with TMA stores.  d = 256 has no room and stores from registers.
  static constexpr bool kStageO = !kWide;
  static constexpr int kOChunks = D * 2 / 128 > 0 ? D * 2 / 128 : 1;
  static constexpr int kOOff = kRingOff + kSlots * kTileBytes;
  static constexpr int kOBytes = kStageO ? kTile * D * 2 : 0;
  // Exchange between the two softmax warpgroups: row maxima
  // [2 parity][2 warpgroups][128 rows], then row sums [2][2][128].
  static constexpr int kXOff = kOOff + kOBytes;
  static constexpr int kXBytes = 2 * 2 * 2 * kTile * 4;
  // 128 x 16 tile of ones (unswizzled K-major core matrices): B operand of
  // the row-sum product L += P 1.
  static constexpr int kOnesOff = kXOff + kXBytes;
  static constexpr int kOnesBytes = kTile * 16 * 2;
  static constexpr int kBarOff = kOnesOff + kOnesBytes;
  // q_full, q_tmem, kv_full[kSlots], kv_empty[kSlots], s_full[2], p_full[2], pv_done, o_full, mma_done,
  // xmax[2], xsum, o_free, o_staged
  static constexpr int kNumBars = 2 + 2 * kSlots + 12;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // The CTA's first kTabSlots work units, decoded once at set-up (two int4
  // per slot; see unit_of), so that no role spends the time at a tile
  // boundary on the integer divisions of the decode.
  static constexpr int kTabSlots = 256;
  static constexpr int kTabOff = kMiscOff + 16;
  static constexpr int kBytes = kTabOff + kTabSlots * 32;
  static constexpr int kAlloc = kBytes + 1024 <= 232448 ? kBytes + 1024 : 232448;
  static_assert(kBytes <= 232448, "shared memory budget");
  // Tensor-memory columns.  d = 256: the two S buffers and O take all 512
  // columns, so Q stays in shared memory (S = Q K^T reads both operands
  // from there) and the row sums of the 16-bit P are added up by the softmax
  // threads instead of a row-sum MMA.
  static constexpr uint32_t kColQ = 0;
  static constexpr uint32_t kColS = kWide ? 0 : 64;    // buffer b at kColS + 128 b
  static constexpr uint32_t kColO = kWide ? 256 : 320;
  static constexpr uint32_t kColL = kColO + D;  // 16 columns: row sums of the 16-bit P (d <= 128)
  static_assert(kWide ? kColO + D <= 512 : kColL + 16 <= 512, "tensor memory budget");
  static_assert(!F8 || D == 128, "the 8-bit forward is built for d = 128");
};

// F8: Q, K, V are E4M3 with per-tensor descale factors.  scale_log2 then
// carries scale * descale_q * descale_k * log2(e), o_scale = descale_v
// multiplies O in the epilogue, P is rounded to E4M3 for O += P V (and for
// its row sums), both products run as kind::f8f6f4, and O is written as bf16
// (BF16 = true).  The 16-bit kernels ignore o_scale.
template <int D, bool BF16, bool CAUSAL, bool F8 = false>
__global__ void __launch_bounds__(384, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               uint16_t* __restrict__ o_ptr,
               float* __restrict__ lse_ptr, const int* __restrict__ cu_q, const int* __restrict__ cu_k, int H,
               int Nq, int Nk, int bottom_right, float scale_log2, int problems, int grid_tiles, int group,
               int fold, float o_scale) {
  static_assert(!F8 || BF16, "the 8-bit forward writes bf16");
  using L = FwdLayout<D, F8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* q_tmem = bars + 1;
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = kv_full + L::kSlots;
  uint64_t* s_full = kv_empty + L::kSlots;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_full = pv_done + 1;
  uint64_t* mma_done = o_full + 1;
  uint64_t* xmax_bar = mma_done + 1;  // [2], 256 arrivals each
  uint64_t* xsum_bar = xmax_bar + 2;  // 256 arrivals
  uint64_t* o_free = xsum_bar + 1;    // the O staging tile may be written (thread 128 arrives)
  uint64_t* o_staged = o_free + 1;    // 256 arrivals: the O tile is staged
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  float* xchg = reinterpret_cast<float*>(smem + L::kXOff);                 // [2 parity][2 wg][128]
  float* xsum = reinterpret_cast<float*>(smem + L::kXOff + L::kXBytes / 2);  // [2 sums][2 wg][128]

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // Work units.  A unit is one 128-row query tile of one problem: slab z of
  // the tensor maps ([z][Nq or Nk][D]) and rows [q0, q0 + nq) / [k0, k0 + nk)
  // of it.  Dense batches have one slab per (batch, head) and use all of it;
  // packed variable-length batches have one slab per head and take sequence
  // b's rows from the offsets, clamped to the slab (bad offsets can give
  // wrong values but never address outside the tensors).  The grid is
  // persistent (at most one CTA per SM) and deals the units of the launch
  // order of tile_order.h (grid_tiles query tiles of each of `problems`
  // problems, causal grids heaviest first) out by unit_at: the units in
  // flight at any time are neighbours in that order, and with `fold` (causal
  // grids) a CTA takes a heavy tile and a light one together.  Every role
  // walks the same units and takes the same decisions.
  const UnitPlan plan = unit_plan(problems, grid_tiles, group, fold);
  const int slots = unit_slots(plan, gridDim.x);
  auto unit_index = [&](int s) { return unit_at(plan, gridDim.x, blockIdx.x, s); };
  struct Unit {
    int z, q0, k0, nq, nk, qt, n, off;
    bool live;  // false: past the end of a shorter sequence, nothing to do
  };
  auto unit_of = [&](int u) {
    Unit w;
    int px, ty;
    grouped_order(static_cast<unsigned>(u), problems, grid_tiles, group, &px, &ty);
    w.z = px;
    w.q0 = 0;
    w.k0 = 0;
    w.nq = Nq;
    w.nk = Nk;
    if (cu_q != nullptr) {
      const int b = px / H;
      w.z = px - b * H;
      auto clamp = [](int v, int hi) { return v < 0 ? 0 : (v > hi ? hi : v); };
      w.q0 = clamp(cu_q[b], Nq);
      w.k0 = clamp(cu_k[b], Nk);
      w.nq = clamp(cu_q[b + 1], Nq) - w.q0;
      w.nk = clamp(cu_k[b + 1], Nk) - w.k0;
      w.nq = w.nq < 0 ? 0 : w.nq;
      w.nk = w.nk < 0 ? 0 : w.nk;
    }
    const int nqt = (w.nq + kTile - 1) / kTile;  // the last tiles may be ragged
    const int nkt = (w.nk + kTile - 1) / kTile;
    w.live = ty < nqt;
    // Causal: the heaviest query tiles come first.
    w.qt = CAUSAL ? (nqt - 1 - ty) : ty;
    // Key tiles this query tile sees.  Causal: query i sees key k iff
    // k <= i + off (off = 0 top-left, nk - nq bottom-right).
    w.off = bottom_right ? w.nk - w.nq : 0;
    w.n = nkt;
    if (CAUSAL && w.live) {
      const int last_row = w.qt * kTile + kTile - 1 < w.nq - 1 ? w.qt * kTile + kTile - 1 : w.nq - 1;
      const int last_key = last_row + w.off < w.nk - 1 ? last_row + w.off : w.nk - 1;
      w.n = last_key < 0 ? 0 : last_key / kTile + 1;
    }
    return w;
  };
  // Slot r's unit: false for an empty slot.  Slots below kTabSlots come from
  // the table (n = -1 marks a unit past the end of a shorter sequence, -2 an
  // empty slot), later ones are decoded here.
  int4* tab = reinterpret_cast<int4*>(smem + L::kTabOff);
  auto slot_unit = [&](int r, Unit& w) {
    if (r < L::kTabSlots) {
      const int4 a = tab[2 * r], c = tab[2 * r + 1];
      if (c.z == -2) return false;
      w.z = a.x; w.q0 = a.y; w.k0 = a.z; w.nq = a.w;
      w.nk = c.x; w.qt = c.y; w.n = c.z < 0 ? 0 : c.z; w.off = c.w;
      w.live = c.z != -1;
      return true;
    }
    const int u = unit_index(r);
    if (u < 0) return false;
    w = unit_of(u);
    return true;
  };

  // Refuse to run (and report) if alignment left too little shared memory.
  if (static_cast<uint32_t>(smem - smem_raw) + L::kBytes > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) atomicExch(&g_device_status, kStatusSmem);
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_tmem, 256);
    for (int i = 0; i < L::kSlots; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 256);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(mma_done, 1);
    mbar_init(&xmax_bar[0], 256);
    mbar_init(&xmax_bar[1], 256);
    mbar_init(xsum_bar, 256);
    mbar_init(o_free, 1);
    mbar_init(o_staged, 256);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 3) {
    const uint32_t one2 = F8 ? 0x38383838u : (BF16 ? 0x3F803F80u : 0x3C003C00u);  // ones (E4M3 or 16-bit)
    uint4* ones = reinterpret_cast<uint4*>(smem + L::kOnesOff);
    for (int i = lane; i < L::kOnesBytes / 16; i += 32) ones[i] = make_uint4(one2, one2, one2, one2);
    fence_proxy_async_smem();
    // The unit table.
    const int n_tab = slots < L::kTabSlots ? slots : L::kTabSlots;
    for (int r = lane; r < n_tab; r += 32) {
      const int u = unit_index(r);
      if (u < 0) {
        tab[2 * r + 1] = make_int4(0, 0, -2, 0);
        continue;
      }
      const Unit w = unit_of(u);
      tab[2 * r] = make_int4(w.z, w.q0, w.k0, w.nq);
      tab[2 * r + 1] = make_int4(w.nk, w.qt, w.live ? w.n : -1, w.off);
    }
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
      int item = 0;  // ring position over all units
      int uu = 0;    // units with key tiles whose Q load was issued
      bool ok = true;
      for (int r = 0; ok && r < slots; ++r) {
        Unit w;
        if (!slot_unit(r, w) || !w.live || w.n == 0) continue;
        // The Q buffer is free once the previous unit's Q has been copied
        // into tensor memory (d = 256: once its S products are done).
        if (uu > 0 && !(ok = mbar_wait(L::kWide ? o_full : q_tmem, (uu - 1) & 1, abort_flag))) break;
        mbar_arrive_expect_tx(q_full, L::kTileBytes);
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(smem + L::kQOff + c * L::kChunkBytes, &tm_q, q_full, c * L::kChunkElems,
                      w.q0 + w.qt * kTile, w.z);
        ++uu;  // Q loads issued
        // Ring order: K_0, K_1, then V_j, K_{j+2} for j = 0, 1, ...
        auto load = [&](const CUtensorMap* map, int tile) {
          const int slot = item % L::kSlots;
          if (!mbar_wait(&kv_empty[slot], ((item / L::kSlots) & 1) ^ 1, abort_flag)) return false;
          mbar_arrive_expect_tx(&kv_full[slot], L::kTileBytes);
          uint8_t* dst = smem + L::kRingOff + slot * L::kTileBytes;
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_3d(dst + c * L::kChunkBytes, map, &kv_full[slot], c * L::kChunkElems, w.k0 + tile * kTile, w.z);
          ++item;
          return true;
        };
        for (int j = 0; ok && j < 2 && j < w.n; ++j) ok = load(&tm_k, j);
        for (int j = 0; ok && j < w.n; ++j) {
          ok = load(&tm_v, j);
          if (ok && j + 2 < w.n) ok = load(&tm_k, j + 2);
        }
      }
      if (!ok) {
        // Let the copies already issued land before the CTA exits.
        if (uu > 0) mbar_drain(q_full, (uu - 1) & 1);
        const int first = item > L::kSlots ? item - L::kSlots : 0;
        for (int i = first; i < item; ++i) mbar_drain(&kv_full[i % L::kSlots], (i / L::kSlots) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (descriptors stay warp-uniform); one
    // elected lane issues each group of MMAs together with its commits.
    // A = Q (TMEM), B = K K-major; A = P (TMEM), B = V MN-major.
    constexpr uint32_t kIdS = F8 ? idesc_e4m3(128, 128, false, false) : idesc_f16(BF16, 128, 128, false, false);
    constexpr uint32_t kIdPV = F8 ? idesc_e4m3(128, D, false, true) : idesc_f16(BF16, 128, D, false, true);
    const uint32_t ring_base = smem_u32(smem + L::kRingOff);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    int item = 0;  // ring position, same order as the producer
    auto wait_slot = [&](uint32_t& addr) {
      const int slot = item % L::kSlots;
      addr = ring_base + slot * L::kTileBytes;
      return wait_all(&kv_full[slot], (item / L::kSlots) & 1);
    };
    // S = Q K^T: A = Q in TMEM (8 columns per K step of 32 bytes: 16
    // 16-bit or 32 8-bit values), B = K K-major (a K step is 32 bytes inside
    // a 128-byte swizzle row).
    const uint64_t qd = sdesc_sw128(smem_u32(smem + L::kQOff), 16, 1024);
    auto issue_s = [&](int b, uint32_t k_addr) {
      const uint64_t kd = sdesc_sw128(k_addr, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < L::kRowBytes / 32; ++ks) {
        const uint32_t step = (ks >> 2) * L::kChunkBytes + (ks & 3) * 32;
        if constexpr (L::kWide)  // A = Q in shared memory
          mma_ss(tmem + L::kColS + 128 * b, qd + (step >> 4), kd + (step >> 4), kIdS, ks > 0 ? 1u : 0u);
        else if constexpr (F8)
          mma_ts_f8(tmem + L::kColS + 128 * b, tmem + L::kColQ + 8 * ks, kd + (step >> 4), kIdS, ks > 0 ? 1u : 0u);
        else
          mma_ts(tmem + L::kColS + 128 * b, tmem + L::kColQ + 8 * ks, kd + (step >> 4), kIdS, ks > 0 ? 1u : 0u);
      }
    };
    // O += P V: P in the buffer's TMEM columns (a key step of kKeysPerStep
    // keys takes 8 columns; the keys of warpgroup h start at column 64 h),
    // V MN-major (kKeysPerStep rows of 128 bytes per step); then L += P 1
    // against the ones tile (two 256-byte core matrices per step).
    constexpr uint32_t kIdL = F8 ? idesc_e4m3(128, 16, false, false) : idesc_f16(BF16, 128, 16, false, false);
    constexpr int kHalfSteps = 64 / L::kKeysPerStep;  // key steps per warpgroup half of a tile
    const uint64_t ones_d = sdesc_noswz(smem_u32(smem + L::kOnesOff), 256, 128);
    auto issue_pv = [&](int b, uint32_t v_addr, bool acc) {
      const uint64_t vd = sdesc_sw128(v_addr, L::kChunkBytes, 1024);
#pragma unroll
      for (int ks = 0; ks < kTile / L::kKeysPerStep; ++ks) {
        const uint32_t p_col = tmem + L::kColS + 128 * b + 64 * (ks / kHalfSteps) + 8 * (ks % kHalfSteps);
        const uint64_t v_step = vd + 8 * L::kKeysPerStep * ks;  // kKeysPerStep rows of 128 bytes, in 16-byte units
        if constexpr (F8)
          mma_ts_f8(tmem + L::kColO, p_col, v_step, kIdPV, (acc || ks > 0) ? 1u : 0u);
        else
          mma_ts(tmem + L::kColO, p_col, v_step, kIdPV, (acc || ks > 0) ? 1u : 0u);
      }
      if constexpr (!L::kWide) {
#pragma unroll
        for (int ks = 0; ks < kTile / L::kKeysPerStep; ++ks) {
          const uint32_t p_col = tmem + L::kColS + 128 * b + 64 * (ks / kHalfSteps) + 8 * (ks % kHalfSteps);
          if constexpr (F8)
            mma_ts_f8(tmem + L::kColL, p_col, ones_d + 32 * ks, kIdL, (acc || ks > 0) ? 1u : 0u);
          else
            mma_ts(tmem + L::kColL, p_col, ones_d + 32 * ks, kIdL, (acc || ks > 0) ? 1u : 0u);
        }
      }
    };

    // Key tiles run through the two S buffers in turn over all units: the
    // g-th key tile of this CTA uses buffer g & 1.
    int uu = 0, g = 0;  // units with key tiles, key tiles before the current unit
    bool ok = true;
    for (int r = 0; ok && r < slots; ++r) {
      Unit w;
      if (!slot_unit(r, w) || !w.live || w.n == 0) continue;
      const int n = w.n;
      // Q of this unit is in tensor memory (d = 256: in shared memory).
      if (!(ok = wait_all(q_tmem, uu & 1))) break;
      for (int j = 0; ok && j < 2 && j < n; ++j) {
        uint32_t ka;
        if (!(ok = wait_slot(ka))) break;
        tc_fence_after();
        if (elect_one()) {
          issue_s((g + j) & 1, ka);
          mma_commit(&s_full[(g + j) & 1]);
          mma_commit(&kv_empty[item % L::kSlots]);
        }
        __syncwarp();
        ++item;
      }
      for (int j = 0; ok && j < n; ++j) {
        const int b = (g + j) & 1;
        uint32_t va;
        if (!(ok = wait_slot(va))) break;
        if (!(ok = wait_all(&p_full[b], ((g + j) >> 1) & 1))) break;
        tc_fence_after();
        if (elect_one()) {
          // j = 0 starts the unit's O and L afresh; the previous unit's
          // epilogue has read them (its p_full follows that epilogue).
          issue_pv(b, va, j > 0);
          mma_commit(pv_done);
          mma_commit(&kv_empty[item % L::kSlots]);
          if (j == n - 1) mma_commit(o_full);
        }
        __syncwarp();
        ++item;
        if (j + 2 < n) {
          uint32_t ka;
          if (!(ok = wait_slot(ka))) break;
          tc_fence_after();
          if (elect_one()) {
            issue_s(b, ka);  // P(j) in this buffer was consumed by PV(j) above
            mma_commit(&s_full[b]);
            mma_commit(&kv_empty[item % L::kSlots]);
          }
          __syncwarp();
          ++item;
        }
      }
      g += n;
      ++uu;
    }
    if (elect_one()) mma_commit(mma_done);
    __syncwarp();
    mbar_drain(mma_done, 0);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int h = (warp - 4) >> 2;   // key columns [64h, 64h + 64) of each tile
    const int wq = warp & 3;         // 32-lane TMEM slice of this warp
    const int row = wq * 32 + lane;  // query row within the tile
    const uint32_t t_row = tmem + (static_cast<uint32_t>(wq * 32) << 16);

    const bool pos_scale = scale_log2 > 0.f;
    const float cx = pos_scale ? scale_log2 : 1.f;
    int uu = 0, g = 0;  // units with key tiles, key tiles before the current unit
    int ot = 0;         // O tiles staged so far
    // Q -> TMEM: this thread copies its row's half of the head dimension
    // (16-byte units of the 128-byte swizzled tile) as 32-bit words of two
    // 16-bit or four 8-bit values, the lowest K index in the lowest bits
    // (d = 256: Q stays in shared memory; only the handshake remains).
    auto copy_q = [&](uint32_t parity) {
      const bool landed = __all_sync(0xffffffffu, mbar_wait(q_full, parity, abort_flag));
      if constexpr (!L::kWide) {
        if (landed) {
          constexpr bool kTwoChunks = L::kRowBytes == 256;  // each warpgroup copies one whole chunk
          constexpr int kUnits = L::kRowBytes / 32;          // 16-byte units in half a row
          const uint8_t* qrow = smem + L::kQOff + (kTwoChunks ? h * L::kChunkBytes : 0) + row * 128;
          uint32_t qv[4 * kUnits];
#pragma unroll
          for (int e = 0; e < kUnits; ++e) {
            const int unit = (kTwoChunks ? e : kUnits * h + e) ^ (row & 7);
            const uint4 v4 = *reinterpret_cast<const uint4*>(qrow + unit * 16);
            qv[4 * e] = v4.x; qv[4 * e + 1] = v4.y; qv[4 * e + 2] = v4.z; qv[4 * e + 3] = v4.w;
          }
          if constexpr (kTwoChunks) {
            tmem_st32(t_row + L::kColQ + 32 * h, qv);
          } else {
            tmem_st16(t_row + L::kColQ + 16 * h, qv);
          }
          tmem_st_wait();
          tc_fence_before();
        }
      }
      mbar_arrive(q_tmem);
      return landed;
    };
    bool q_ready = false;  // the next unit's Q is already in tensor memory
    bool ok = true;
    for (int r = 0; ok && r < slots; ++r) {
      Unit w;
      if (!slot_unit(r, w) || !w.live) continue;
      const int z = w.z, q0 = w.q0, nq = w.nq, nk = w.nk, qt = w.qt, n = w.n, off = w.off;
      if (n == 0) {
        // No row of this tile sees a key (bottom-right with nq > nk, or a
        // sequence without keys): the softmax is empty, O = 0 and LSE = log 0.
        const int rows = nq - qt * kTile < kTile ? nq - qt * kTile : kTile;
        const size_t grow0 = static_cast<size_t>(z) * Nq + q0 + static_cast<size_t>(qt) * kTile;
        const int t0 = static_cast<int>(threadIdx.x) - 128;  // the 256 softmax threads
        for (int e = t0; e < rows * D / 8; e += 256)
          reinterpret_cast<uint4*>(o_ptr + grow0 * D)[e] = make_uint4(0u, 0u, 0u, 0u);
        for (int e = t0; e < rows; e += 256) lse_ptr[grow0 + e] = -INFINITY;
        continue;
      }
      if (!q_ready) ok = copy_q(uu & 1);
      q_ready = false;

      float m_run = -INFINITY;  // running row max (log2 units; stale by < 8)
      float l_run = 0.f;        // this warpgroup's part of sum exp2(score - m_run)
      float lr_run = 0.f;       // d = 256: the same sum of the 16-bit rounded values

      for (int j = 0; ok && j < n; ++j) {
        const int gj = g + j;  // key tile count over all units of this CTA
        const int b = gj & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (gj >> 1) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint32_t s_col = t_row + L::kColS + 128 * b + 64 * h;
        float x[64];
        {
          uint32_t r[64];
          tmem_ld64(s_col, r);
#pragma unroll
          for (int i = 0; i < 64; ++i) x[i] = __uint_as_float(r[i]);
        }
        if (!pos_scale) {
#pragma unroll
          for (int c = 0; c < 64; ++c) x[c] *= scale_log2;
        }
        // Mask keys past nk (ragged last tile) and, causal, keys after
        // query + off: column c is kept iff c <= lim.
        const int kv_valid = nk - j * kTile;
        const int diag_lim = (qt - j) * kTile + off;  // lim of row 0 from the mask
        if ((CAUSAL && diag_lim < kTile - 1) || kv_valid < kTile) {
          int lim = kv_valid - 1;
          if (CAUSAL && diag_lim + row < lim) lim = diag_lim + row;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (64 * h + c > lim) x[c] = -INFINITY;
        }
        float mp[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mp[i] = x[i];
#pragma unroll
        for (int c = 8; c < 64; c += 2) mp[(c >> 1) & 7] = max3f(mp[(c >> 1) & 7], x[c], x[c + 1]);
        float mx = max3f(max3f(mp[0], mp[1], mp[2]), max3f(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
        // Exponentials, sums and the in-place 16-bit P of this warpgroup's 64
        // columns against the maximum m_run.  l_run sums the fp32
        // probabilities (for LSE); the tensor core sums the rounded 16-bit ones
        // (L).  Arguments and sums as packed fp32x2; one pair in four goes to
        // the FMA-pipe exponential, since MUFU throughput bounds them otherwise.
        // A row that has seen no key yet (m_run = -inf; causal with off < 0)
        // uses 0: its scores are all -inf, so p = 0 rather than NaN.
        // (d = 256: the rounded ones are summed here too, in sr.  F8: P is
        // rounded to E4M3, four keys per 32-bit column, so the 64 keys take
        // 16 columns; the lazy rescale keeps P <= 2^8, inside E4M3's 448.)
        float2 su[4], sr[4];
  #define ATTN_EXP_STORE()                                                                            \
    {                                                                                                 \
      _Pragma("unroll") for (int i = 0; i < 4; ++i) su[i] = sr[i] = make_float2(0.f, 0.f);            \
      const float m_use = m_run == -INFINITY ? 0.f : m_run;                                           \
      const float2 cx2 = make_float2(cx, cx), negm2 = make_float2(-m_use, -m_use);                    \
      if constexpr (F8) {                                                                             \
        uint32_t pk[16];                                                                              \
        _Pragma("unroll") for (int i = 0; i < 16; ++i) {                                              \
          const float2 a0 = fma2(make_float2(x[4 * i], x[4 * i + 1]), cx2, negm2);                    \
          const float2 a1 = fma2(make_float2(x[4 * i + 2], x[4 * i + 3]), cx2, negm2);                \
          const float2 p0 = make_float2(ex2(a0.x), ex2(a0.y));                                        \
          const float2 p1 = (i & 1) ? exp2_poly2(a1) : make_float2(ex2(a1.x), ex2(a1.y));             \
          pk[i] = pack4_e4m3(p0.x, p0.y, p1.x, p1.y);                                                 \
          su[(2 * i) & 3] = add2(su[(2 * i) & 3], p0);                                                \
          su[(2 * i + 1) & 3] = add2(su[(2 * i + 1) & 3], p1);                                        \
        }                                                                                             \
        tmem_st16(s_col, pk);                                                                         \
      } else {                                                                                        \
      _Pragma("unroll") for (int c = 0; c < 2; ++c) {                                                 \
        uint32_t pk[16];                                                                              \
        _Pragma("unroll") for (int i = 0; i < 16; ++i) {                                              \
          const float2 a = fma2(make_float2(x[32 * c + 2 * i], x[32 * c + 2 * i + 1]), cx2, negm2);   \
          const float2 p = ((i & 3) == 3) ? exp2_poly2(a) : make_float2(ex2(a.x), ex2(a.y));          \
          pk[i] = pack2<BF16>(p.x, p.y);                                                              \
          su[i & 3] = add2(su[i & 3], p);                                                             \
          if constexpr (L::kWide) sr[i & 3] = add2(sr[i & 3], unpack2<BF16>(pk[i]));                  \
        }                                                                                             \
        tmem_st16(s_col + 16 * c, pk);                                                                \
      }                                                                                               \
      }                                                                                               \
    }
        // Row maximum over both halves of the key tile, exchanged through
        // shared memory (double-buffered by tile parity: a warpgroup cannot
        // rewrite a slot before the other has passed the next exchange, which
        // it reaches only after reading the slot).
        xchg[(b * 2 + h) * kTile + row] = mx;
        mbar_arrive(&xmax_bar[b]);
        // After the first tile, compute P against the current maximum while
        // the other warpgroup's half arrives: it stands unless the maximum has
        // grown by more than 2^8 (then it is recomputed below; P is not read
        // before p_full).
        if (j > 0) ATTN_EXP_STORE()
        ok = __all_sync(0xffffffffu, mbar_wait(&xmax_bar[b], (gj >> 1) & 1, abort_flag));
        if (!ok) break;
        mx = fmaxf(mx, xchg[(b * 2 + (h ^ 1)) * kTile + row]);
        const float m_new = fmaxf(m_run, mx * cx);
        // Rescale O and the sums only when the maximum has grown by more than
        // 2^8; otherwise keep the stale maximum (P stays below 256).  Both
        // warpgroups see the same m_run and m_new, so they decide alike.
        const bool need = (j > 0) && (m_new - m_run > 8.f);
        if (j == 0) m_run = m_new;
        const bool any_need = __any_sync(0xffffffffu, need);
        if (any_need) {
          // O must hold PV(j-1) complete before it is rescaled.
          ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (gj - 1) & 1, abort_flag));
          if (!ok) break;
          tc_fence_after();
          const float alpha = need ? ex2(m_run - m_new) : 1.f;
#pragma unroll 1
          for (int c = 0; c < D / 64; ++c) {
            uint32_t r[32];
            tmem_ld32(t_row + L::kColO + (D / 2) * h + 32 * c, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(t_row + L::kColO + (D / 2) * h + 32 * c, r);
          }
          if constexpr (!L::kWide) {
            if (h == 0) tmem_st1(t_row + L::kColL, __float_as_uint(__uint_as_float(tmem_ld1(t_row + L::kColL)) * alpha));
          }
          if (need) {
            l_run *= alpha;
            lr_run *= alpha;
            m_run = m_new;
          }
        }
        // First tile, or a maximum that moved: (re)compute against the final
        // m_run (rows of the warp whose m_run did not move get the same values).
        if (j == 0 || any_need) {
          if (j > 0) tmem_st_wait();  // the optimistic stores land before they are overwritten
          ATTN_EXP_STORE()
        }
  #undef ATTN_EXP_STORE
        const float2 su01 = add2(su[0], su[1]), su23 = add2(su[2], su[3]);
        l_run += (su01.x + su01.y) + (su23.x + su23.y);
        if constexpr (L::kWide) {
          const float2 sr01 = add2(sr[0], sr[1]), sr23 = add2(sr[2], sr[3]);
          lr_run += (sr01.x + sr01.y) + (sr23.x + sr23.y);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[b]);
      }
      // The next unit's Q goes into tensor memory now, before this unit's
      // epilogue: every S product of this unit (the readers of the old Q)
      // has been consumed, and the MMA warp can start the next unit's first
      // two S products while the epilogue runs (d <= 128; at d = 256 the
      // next Q is loaded only once this unit's products are done).
      if constexpr (!L::kWide) {
        for (int r2 = r + 1; ok && r2 < slots; ++r2) {
          Unit w2;
          if (!slot_unit(r2, w2) || !w2.live || w2.n == 0) continue;
          ok = copy_q((uu + 1) & 1);
          q_ready = true;
          break;
        }
      }
      // Epilogue: combine the two warpgroups' row sums, then each warpgroup
      // writes its half of the head dimension of O.
      xsum[h * kTile + row] = l_run;
      if constexpr (L::kWide) xsum[(2 + h) * kTile + row] = lr_run;
      mbar_arrive(xsum_bar);
      if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(xsum_bar, uu & 1, abort_flag));
      if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(o_full, uu & 1, abort_flag));
      if (ok && n > 0) {
        tc_fence_after();
        const float l_tot = l_run + xsum[(h ^ 1) * kTile + row];
        // A row that sees no key keeps m_run = -inf: O = 0 and LSE = -inf.
        // (Its sums are not exactly 0: the FMA-pipe exponential returns
        // ~2^-126 rather than 0 for a masked score.)
        // (tcgen05.ld is warp-collective: every lane loads, then selects.)
        const bool empty = m_run == -INFINITY;
        float l_tc;
        if constexpr (L::kWide)
          l_tc = lr_run + xsum[(2 + (h ^ 1)) * kTile + row];
        else
          l_tc = __uint_as_float(tmem_ld1(t_row + L::kColL));
        const float inv = empty ? 0.f : (F8 ? o_scale : 1.f) / l_tc;
        const bool live = qt * kTile + row < nq;  // padding rows of a ragged tile are not stored
        const size_t grow = static_cast<size_t>(z) * Nq + q0 + static_cast<size_t>(qt) * kTile + row;
        // O leaves through the staging tile and TMA stores (rows past the
        // map's extent are not written) for dense batches and for full tiles
        // of packed ones; a ragged tile of a packed batch stores its live rows
        // from registers, so that it never touches the next sequence's rows.
        // Thread 128 issues the stores; it lets the tile be rewritten once
        // its previous stores have read it (o_free), and stores it once
        // every softmax thread has staged its part (o_staged).
        const bool staged = L::kStageO && (cu_q == nullptr || qt * kTile + kTile <= nq);
        if (staged) {
          if (threadIdx.x == 128) {
            tma_store_wait_read();
            mbar_arrive(o_free);
          }
          ok = __all_sync(0xffffffffu, mbar_wait(o_free, ot & 1, abort_flag));
        }
        uint4* dst = reinterpret_cast<uint4*>(o_ptr + grow * D + (D / 2) * h);
#pragma unroll 1
        for (int c = 0; ok && c < D / 64; ++c) {
          uint32_t r[32];
          tmem_ld32(t_row + L::kColO + (D / 2) * h + 32 * c, r);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack2<BF16>(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
          if (staged) {
            // 16-byte unit u of the row (columns 8u .. 8u+7) sits in chunk
            // u / 8 at swizzled position (u % 8) ^ (row % 8).
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int u = D * h / 16 + 4 * c + v;
              *reinterpret_cast<uint4*>(smem + L::kOOff + (u / 8) * L::kChunkBytes + row * 128 +
                                        (((u % 8) ^ (row & 7)) * 16)) =
                  make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
          } else if (live) {
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
        if (staged) {
          fence_proxy_async_smem();
          mbar_arrive(o_staged);
          if (threadIdx.x == 128 && mbar_wait(o_staged, ot & 1, abort_flag)) {
            for (int c = 0; c < L::kOChunks; ++c)
              tma_store_3d(&tm_o, smem + L::kOOff + c * L::kChunkBytes, c * 64, q0 + qt * kTile, z);
            tma_store_commit();
          }
          ++ot;
        }
        if (h == 0 && live) lse_ptr[grow] = empty ? -INFINITY : (m_run + lg2(l_tot)) * 0.69314718055994530942f;
      }
      g += n;
      ++uu;
    }
    // The last O stores have landed before the CTA (and its shared memory) ends.
    if (threadIdx.x == 128) tma_store_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn
