// fwd_kernel.cuh -- fused attention forward for sm_100a.
//
// Computes, for one (batch, head) slice and a pair of 128-row query tiles,
//   S = Q K^T (tcgen05 MMA into tensor memory), the online softmax over the
//   key tiles (running row maximum m and row sum l, rescaling with exp2),
//   P cast to 16-bit in tensor memory, O += P V (tcgen05 MMA with P read from
//   tensor memory), and the epilogue O / l and LSE = ln2 * (m + log2 l).
// This is the tiled, fused algorithm of the page "FlashAttention 核心原理"
// (part 2, tiling and kernel fusion) with the online softmax named on the
// page "Flash Attention 落地评估" (section 4); S never leaves the SM.
//
// CTA layout (384 threads, one CTA per SM):
//   warp 0       TMA producer: both Q tiles once, then K_j, V_j through a
//                ring of shared-memory slots
//   warp 1       MMA issuer (one thread): S_t = Q_t K_j^T, O_t += P_t V_j
//   warp 2       tensor-memory allocation / release
//   warps 4-7    softmax for query tile 0   (thread = query row = TMEM lane)
//   warps 8-11   softmax for query tile 1
// The two query tiles ping-pong: while one warpgroup exponentiates its
// scores, the tensor core works on the other tile.
//
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   [0,128) S_0 (P_0 packed 16-bit in [0,64)), [128,256) S_1 (P_1),
//   [256,256+D) O_0, [256+D,256+2D) O_1.
#pragma once

#include "sm100.cuh"

namespace attn {

constexpr int kTile = 128;  // rows of a query tile and of a key/value tile

template <int D>
struct FwdLayout {
  static constexpr int kChunks = D / 64;            // 128-byte column chunks per row
  static constexpr int kChunkBytes = kTile * 128;   // one 128-row chunk
  static constexpr int kTileBytes = kTile * D * 2;  // one 128 x D 16-bit tile
  static constexpr int kSlots = D == 128 ? 5 : 8;   // K/V ring slots
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = kQOff + 2 * kTileBytes;
  static constexpr int kBarOff = kRingOff + kSlots * kTileBytes;
  // q_full, kv_full[kSlots], kv_empty[kSlots], s_full[2], p_full[2], o_full[2], mma_done
  static constexpr int kNumBars = 1 + 2 * kSlots + 7;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
  static_assert(kAlloc <= 232448, "shared memory budget");
};

template <int D, bool BF16, bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ o_ptr,
               float* __restrict__ lse_ptr, int Nq, int Nk, float scale_log2, int num_pairs) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + L::kSlots;
  uint64_t* s_full = kv_empty + L::kSlots;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* mma_done = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int bh = blockIdx.x;
  // Causal: the heaviest query-tile pairs are launched first.
  const int pair = CAUSAL ? (num_pairs - 1 - static_cast<int>(blockIdx.y)) : static_cast<int>(blockIdx.y);
  const int nqt = Nq / kTile;
  const int nkt = Nk / kTile;
  int n_kv[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qt = 2 * pair + t;
    n_kv[t] = qt < nqt ? (CAUSAL ? qt + 1 : nkt) : 0;
  }
  const int nkv = n_kv[0] > n_kv[1] ? n_kv[0] : n_kv[1];
  const int ntiles = n_kv[1] > 0 ? 2 : 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < L::kSlots; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_full[t], 1);
    }
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
      const int qrow0 = bh * Nq + 2 * pair * kTile;
      mbar_arrive_expect_tx(q_full, ntiles * L::kTileBytes);
      for (int t = 0; t < ntiles; ++t)
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_2d(smem + L::kQOff + t * L::kTileBytes + c * L::kChunkBytes, &tm_q, q_full, c * 64,
                      qrow0 + t * kTile);
      const int krow0 = bh * Nk;
      int item = 0;
      bool ok = true;
      for (int j = 0; j < nkv && ok; ++j) {
        for (int which = 0; which < 2; ++which, ++item) {
          const int slot = item % L::kSlots;
          const uint32_t ph = (item / L::kSlots) & 1;
          if (!mbar_wait(&kv_empty[slot], ph ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&kv_full[slot], L::kTileBytes);
          uint8_t* dst = smem + L::kRingOff + slot * L::kTileBytes;
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_2d(dst + c * L::kChunkBytes, which ? &tm_v : &tm_k, &kv_full[slot], c * 64,
                        krow0 + j * kTile);
        }
      }
      if (!ok) {
        // Let the copies already issued land before the CTA exits.
        mbar_drain(q_full, 0);
        const int first = item > L::kSlots ? item - L::kSlots : 0;
        for (int i = first; i < item; ++i) mbar_drain(&kv_full[i % L::kSlots], (i / L::kSlots) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_f16(BF16, 128, 128, false, false);
      constexpr uint32_t kIdPV = idesc_f16(BF16, 128, D, false, true);
      const uint32_t q_base = smem_u32(smem + L::kQOff);
      const uint32_t ring_base = smem_u32(smem + L::kRingOff);
      auto slot_addr = [&](int item) { return ring_base + (item % L::kSlots) * L::kTileBytes; };
      auto slot_of = [&](int item) { return item % L::kSlots; };
      auto ph_of = [&](int item) { return static_cast<uint32_t>((item / L::kSlots) & 1); };
      // S_t = Q_t K^T: both operands K-major; a K step of 16 elements is 32
      // bytes inside a 128-byte swizzle row, 4 steps per 64-column chunk.
      auto issue_s = [&](int t, uint32_t k_addr) {
        const uint32_t qa = q_base + t * L::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * L::kChunkBytes + (ks & 3) * 32;
          mma_ss(tmem + t * 128, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024), kIdS,
                 ks > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t V: P from TMEM (two 16-bit values per column, 8 columns per
      // K step), V MN-major: a K step of 16 keys is 16 rows of 128 bytes.
      auto issue_pv = [&](int t, uint32_t v_addr, bool acc) {
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks)
          mma_ts(tmem + 256 + t * D, tmem + t * 128 + ks * 8,
                 sdesc_sw128(v_addr + ks * 2048, L::kChunkBytes, 1024), kIdPV, (acc || ks > 0) ? 1u : 0u);
      };

      bool ok = mbar_wait(q_full, 0, abort_flag);
      if (ok && nkv > 0) {
        ok = mbar_wait(&kv_full[slot_of(0)], ph_of(0), abort_flag);
        if (ok) {
          tc_fence_after();
          for (int t = 0; t < 2; ++t)
            if (n_kv[t] > 0) {
              issue_s(t, slot_addr(0));
              mma_commit(&s_full[t]);
            }
          mma_commit(&kv_empty[slot_of(0)]);
        }
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const int vi = 2 * j + 1;  // ring item of V_j
        const int ki = 2 * j + 2;  // ring item of K_{j+1}
        if (!mbar_wait(&kv_full[slot_of(vi)], ph_of(vi), abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        bool k_next = false;
        for (int t = 0; t < 2; ++t) {
          if (j < n_kv[t]) {
            if (!mbar_wait(&p_full[t], j & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(t, slot_addr(vi), j > 0);
            if (j == n_kv[t] - 1) mma_commit(&o_full[t]);
          }
          if (j + 1 < n_kv[t]) {
            if (!k_next) {
              if (!mbar_wait(&kv_full[slot_of(ki)], ph_of(ki), abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              k_next = true;
            }
            issue_s(t, slot_addr(ki));
            mma_commit(&s_full[t]);
          }
        }
        if (!ok) break;
        mma_commit(&kv_empty[slot_of(vi)]);
        if (k_next) mma_commit(&kv_empty[slot_of(ki)]);
      }
      // Every MMA issued above has completed once mma_done flips.
      mma_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;     // query tile of this warpgroup
    const int wq = warp & 3;           // 32-lane TMEM slice of this warp
    const int row = wq * 32 + lane;    // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t s_tm = tmem + lane_off + t * 128;
    const uint32_t o_tm = tmem + lane_off + 256 + t * D;
    const int n = n_kv[t];
    const int qt = 2 * pair + t;
    float m_run = -INFINITY;  // running max of the scores, log2 units (stale by < 8)
    float l_run = 0.f;        // running sum of exp2(score - m_run)
    float l_o = 0.f;          // the same sum over the 16-bit rounded terms
    const bool pos_scale = scale_log2 > 0.f;
    const float cx = pos_scale ? scale_log2 : 1.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      ok = mbar_wait(&s_full[t], j & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // Scores of this row.  With a positive scale, the scale is folded into
      // the exponent's FMA and the maximum is taken on the raw scores;
      // otherwise the scores are scaled first.
      float x[kTile];
#pragma unroll
      for (int c = 0; c < kTile / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(s_tm + c * 32, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[c * 32 + i] = __uint_as_float(r[i]);
      }
      if (!pos_scale) {
#pragma unroll
        for (int c = 0; c < kTile; ++c) x[c] *= scale_log2;
      }
      if (CAUSAL && j == qt) {
#pragma unroll
        for (int c = 0; c < kTile; ++c)
          if (c > row) x[c] = -INFINITY;
      }
      float mp[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mp[i] = x[i];
#pragma unroll
      for (int c = 8; c < kTile; ++c) mp[c & 7] = fmaxf(mp[c & 7], x[c]);
      const float m_tile = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                                 fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7]))) * cx;
      const float m_new = fmaxf(m_run, m_tile);
      // Rescale O and the sums only when the maximum has grown by more than
      // 2^8; otherwise keep the stale maximum (P stays below 256).
      const bool need = (j > 0) && (m_new - m_run > 8.f);
      if (j == 0) m_run = m_new;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? ex2(m_run - m_new) : 1.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(o_tm + c * 32, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(o_tm + c * 32, r);
        }
        if (need) {
          l_run *= alpha;
          l_o *= alpha;
          m_run = m_new;
        }
      }
      // l_run sums the fp32 probabilities (for LSE); l_o sums the rounded
      // 16-bit probabilities that the P V product uses, so that O / l_o is a
      // weighted mean of V rows with weights summing to one.
      float su[4] = {0.f, 0.f, 0.f, 0.f}, sr[4] = {0.f, 0.f, 0.f, 0.f};
      const float neg_m = -m_run;
#pragma unroll
      for (int c = 0; c < kTile / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2(fmaf(x[c * 32 + 2 * i], cx, neg_m));
          const float p1 = ex2(fmaf(x[c * 32 + 2 * i + 1], cx, neg_m));
          pk[i] = pack2<BF16>(p0, p1);
          const float2 pr = unpack2<BF16>(pk[i]);
          su[i & 3] += p0 + p1;
          sr[i & 3] += pr.x + pr.y;
        }
        tmem_st16(s_tm + c * 16, pk);
      }
      l_run += (su[0] + su[1]) + (su[2] + su[3]);
      l_o += (sr[0] + sr[1]) + (sr[2] + sr[3]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    if (ok && n > 0) {
      ok = mbar_wait(&o_full[t], 0, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        const float inv = 1.f / l_o;
        const size_t grow = static_cast<size_t>(bh) * Nq + static_cast<size_t>(qt) * kTile + row;
        uint4* dst = reinterpret_cast<uint4*>(o_ptr + grow * D);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(o_tm + c * 32, r);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack2<BF16>(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
        lse_ptr[grow] = (m_run + lg2(l_run)) * 0.69314718055994530942f;
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
