// host_step.cpp -- forward and backward of a batch held in host memory.
//
// The (batch, head) slices are split into chunks.  The host-to-device copies
// of every chunk run on one internal stream, the attention kernels of each
// chunk on the caller's stream once its inputs have landed, and the
// device-to-host copies of each chunk's results on a second internal stream
// once its kernels are done.  Events chain the three, so the copies of one
// chunk overlap the kernels of another and the two copy directions overlap
// each other.  Nothing here computes: the kernels are the library's own
// attn_fwd and attn_bwd (or attn_bwd_deterministic) on each chunk.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "attn.h"
#include "trace.h"

namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// The two internal copy streams of a device, created on first use and kept
// for the life of the process.
struct CopyStreams {
  cudaStream_t h2d = nullptr;
  cudaStream_t d2h = nullptr;
};

attn_status copy_streams(CopyStreams* out) {
  static std::mutex mu;
  static std::vector<CopyStreams> per_device;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(per_device.size()) <= dev) per_device.resize(dev + 1);
  CopyStreams& s = per_device[dev];
  if (!s.h2d && cudaStreamCreateWithFlags(&s.h2d, cudaStreamNonBlocking) != cudaSuccess) return ATTN_ERR_CUDA;
  if (!s.d2h && cudaStreamCreateWithFlags(&s.d2h, cudaStreamNonBlocking) != cudaSuccess) return ATTN_ERR_CUDA;
  *out = s;
  return ATTN_OK;
}

// Where each tensor sits in the caller's device buffer.  Every region starts
// on a 256-byte boundary; the LSE of each chunk has its own aligned block,
// since the kernels want a 16-byte-aligned LSE and a chunk's first row
// (slice s0 times Nq floats) need not be.
struct Plan {
  long long bh = 0;
  int chunks = 0;
  long long per_chunk = 0;  // slices per chunk (the last may hold fewer)
  size_t q = 0, k = 0, v = 0, dout = 0, o = 0, dq = 0, dk = 0, dv = 0, lse = 0, ws = 0;
  size_t lse_block = 0;     // bytes of one chunk's LSE block
  size_t ws_bytes = 0;
  size_t total = 0;
  size_t eb = 2;            // bytes per element
};

bool make_plan(int B, int H, int Nq, int Nk, int d, int chunks, Plan* p) {
  p->bh = static_cast<long long>(B) * H;
  if (p->bh <= 0 || p->bh > 0x7fffffffLL || Nq <= 0 || Nk <= 0 || d <= 0 || chunks <= 0) return false;
  // The row bounds of the attention calls; they also keep the sizes below far from size_t overflow.
  if (p->bh * Nq > (1LL << 40) || p->bh * Nk > (1LL << 40)) return false;
  p->chunks = static_cast<int>(p->bh < chunks ? p->bh : chunks);
  p->per_chunk = (p->bh + p->chunks - 1) / p->chunks;
  p->chunks = static_cast<int>((p->bh + p->per_chunk - 1) / p->per_chunk);  // no empty chunk
  // Each chunk is one attn_fwd / attn_bwd call with B = 1, H = per_chunk: it
  // must meet their shape rules (tile counts, grid size), checked here so
  // that a shape they would refuse is refused before any copy is enqueued.
  const long long tq = (Nq + 127) / 128, tk = (Nk + 127) / 128;
  if (tq > 65535 || tk > 65535 || p->per_chunk * tq > 0x7fffffffLL || p->per_chunk * tk > 0x7fffffffLL)
    return false;
  const size_t qbytes = static_cast<size_t>(p->bh) * Nq * d * p->eb;
  const size_t kbytes = static_cast<size_t>(p->bh) * Nk * d * p->eb;
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t here = at;
    at += round_up(bytes);
    return here;
  };
  p->q = take(qbytes);
  p->k = take(kbytes);
  p->v = take(kbytes);
  p->dout = take(qbytes);
  p->o = take(qbytes);
  p->dq = take(qbytes);
  p->dk = take(kbytes);
  p->dv = take(kbytes);
  p->lse_block = round_up(static_cast<size_t>(p->per_chunk) * Nq * sizeof(float));
  p->lse = take(p->lse_block * p->chunks);
  p->ws_bytes = attn_bwd_workspace_bytes(1, static_cast<int>(p->per_chunk), Nq, Nk, d);
  if (p->ws_bytes == 0) return false;
  p->ws = take(p->ws_bytes);
  p->total = at;
  return true;
}

// Events of one call: released once the device has passed them.
struct Events {
  std::vector<cudaEvent_t> ev;
  ~Events() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
  }
  cudaEvent_t add() {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    ev.push_back(e);
    return e;
  }
};

// Zeroes dK and dV on the host, in stream order (a problem with no query
// rows has zero key gradients).
struct HostZero {
  void* a;
  void* b;
  size_t bytes;
};

void CUDART_CB zero_host(void* arg) {
  HostZero* z = static_cast<HostZero*>(arg);
  std::memset(z->a, 0, z->bytes);
  std::memset(z->b, 0, z->bytes);
  delete z;
}

}  // namespace

extern "C" {

size_t attn_host_step_device_bytes(int B, int H, int Nq, int Nk, int d, int chunks) {
  Plan p;
  if (!make_plan(B, H, Nq, Nk, d, chunks, &p)) return 0;
  return p.total;
}

attn_status attn_host_step(const void* q_h, const void* k_h, const void* v_h, const void* dout_h, void* o_h,
                           float* lse_h, void* dq_h, void* dk_h, void* dv_h, void* device_buffer,
                           size_t device_bytes, int B, int H, int Nq, int Nk, int d, float scale, int causal,
                           attn_dtype dtype, int chunks, int deterministic, void* stream) {
  attn::TraceRange trace("attn_host_step");
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || d < 0 || chunks < 1) return ATTN_ERR_INVALID_ARG;
  if (causal != ATTN_CAUSAL_NONE && causal != ATTN_CAUSAL_TOP_LEFT && causal != ATTN_CAUSAL_BOTTOM_RIGHT)
    return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_FP16 && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  const long long bh = static_cast<long long>(B) * H;
  if (bh > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (bh == 0) return ATTN_OK;
  if (Nq == 0) {
    // No query rows: dK = dV = 0, written on the host once the caller's
    // stream reaches this call; nothing else.
    if (Nk == 0) return ATTN_OK;
    if (!dk_h || !dv_h) return ATTN_ERR_INVALID_ARG;
    HostZero* z = new HostZero{dk_h, dv_h, static_cast<size_t>(bh) * Nk * d * 2};
    if (cudaLaunchHostFunc(static_cast<cudaStream_t>(stream), zero_host, z) != cudaSuccess) {
      delete z;
      return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
  }
  if (Nk == 0) return ATTN_ERR_INVALID_ARG;  // a softmax over no keys is undefined
  if (!q_h || !k_h || !v_h || !dout_h || !o_h || !lse_h || !dq_h || !dk_h || !dv_h || !device_buffer)
    return ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(device_buffer) % kAlign != 0) return ATTN_ERR_INVALID_ARG;
  Plan p;
  if (!make_plan(B, H, Nq, Nk, d, chunks, &p)) return ATTN_ERR_UNSUPPORTED;
  if (device_bytes < p.total) return ATTN_ERR_INVALID_ARG;

  CopyStreams cs;
  if (copy_streams(&cs) != ATTN_OK) return ATTN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* dev = static_cast<uint8_t*>(device_buffer);
  const size_t qrow = static_cast<size_t>(Nq) * d * p.eb;  // bytes of one slice of Q, dO, O, dQ
  const size_t krow = static_cast<size_t>(Nk) * d * p.eb;  // bytes of one slice of K, V, dK, dV
  Events ev;
  auto fail = [&]() { return ATTN_ERR_CUDA; };

  // The copies start once the caller's stream has reached this call.
  cudaEvent_t start = ev.add();
  if (!start || cudaEventRecord(start, st) != cudaSuccess || cudaStreamWaitEvent(cs.h2d, start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(cs.d2h, start, 0) != cudaSuccess)
    return fail();

  std::vector<cudaEvent_t> in_ready(p.chunks);
  auto h2d = [&](size_t dst, const void* src, size_t off, size_t bytes) {
    return cudaMemcpyAsync(dev + dst + off, static_cast<const uint8_t*>(src) + off, bytes, cudaMemcpyHostToDevice,
                           cs.h2d) == cudaSuccess;
  };
  for (int c = 0; c < p.chunks; ++c) {
    const long long s0 = c * p.per_chunk;
    const long long n = (bh - s0 < p.per_chunk) ? bh - s0 : p.per_chunk;
    const size_t qo = s0 * qrow, ko = s0 * krow, qb = n * qrow, kb = n * krow;
    if (!h2d(p.q, q_h, qo, qb) || !h2d(p.k, k_h, ko, kb) || !h2d(p.v, v_h, ko, kb) || !h2d(p.dout, dout_h, qo, qb))
      return fail();
    in_ready[c] = ev.add();
    if (!in_ready[c] || cudaEventRecord(in_ready[c], cs.h2d) != cudaSuccess) return fail();
  }

  auto d2h = [&](void* dst, size_t src, size_t off, size_t bytes) {
    return cudaMemcpyAsync(static_cast<uint8_t*>(dst) + off, dev + src + off, bytes, cudaMemcpyDeviceToHost,
                           cs.d2h) == cudaSuccess;
  };
  for (int c = 0; c < p.chunks; ++c) {
    const long long s0 = c * p.per_chunk;
    const int n = static_cast<int>((bh - s0 < p.per_chunk) ? bh - s0 : p.per_chunk);
    const size_t qo = s0 * qrow, ko = s0 * krow;
    float* lse_c = reinterpret_cast<float*>(dev + p.lse + c * p.lse_block);
    if (cudaStreamWaitEvent(st, in_ready[c], 0) != cudaSuccess) return fail();
    // One chunk is B = 1, H = n slices (the slices of a [B][H] batch are contiguous).
    attn_status s = attn_fwd(dev + p.q + qo, dev + p.k + ko, dev + p.v + ko, dev + p.o + qo, lse_c, 1, n, Nq, Nk, d,
                             scale, causal, dtype, st);
    if (s != ATTN_OK) return s;
    auto bwd = deterministic ? attn_bwd_deterministic : attn_bwd;
    s = bwd(dev + p.q + qo, dev + p.k + ko, dev + p.v + ko, dev + p.o + qo, lse_c, dev + p.dout + qo, dev + p.dq + qo,
            dev + p.dk + ko, dev + p.dv + ko, dev + p.ws, 1, n, Nq, Nk, d, scale, causal, dtype, st);
    if (s != ATTN_OK) return s;
    cudaEvent_t done = ev.add();
    if (!done || cudaEventRecord(done, st) != cudaSuccess || cudaStreamWaitEvent(cs.d2h, done, 0) != cudaSuccess)
      return fail();
    const size_t qb = static_cast<size_t>(n) * qrow, kb = static_cast<size_t>(n) * krow;
    if (!d2h(o_h, p.o, qo, qb) || !d2h(dq_h, p.dq, qo, qb) || !d2h(dk_h, p.dk, ko, kb) || !d2h(dv_h, p.dv, ko, kb))
      return fail();
    if (cudaMemcpyAsync(lse_h + s0 * Nq, lse_c, static_cast<size_t>(n) * Nq * sizeof(float), cudaMemcpyDeviceToHost,
                        cs.d2h) != cudaSuccess)
      return fail();
  }

  // The caller's stream continues once the last result has reached the host.
  cudaEvent_t end = ev.add();
  if (!end || cudaEventRecord(end, cs.d2h) != cudaSuccess || cudaStreamWaitEvent(st, end, 0) != cudaSuccess)
    return fail();
  return ATTN_OK;
}

}  // extern "C"
