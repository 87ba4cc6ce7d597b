// C ABI of the library (declared in include/tm.h): argument validation, the
// layer schedule, host exports of the static tile list, and status handling.
// All device work is delegated to tm_attn.cu.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <vector>

#include "tm.h"
#include "tm_internal.h"
#include "tm_tiles.cuh"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, long long abytes, const void* b, long long bbytes) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + static_cast<uintptr_t>(bbytes) && b0 < a0 + static_cast<uintptr_t>(abytes);
}

int validate_common(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv,
                    int N, int D, float scale) {
  if (!q || !k || !v || !o) return TM_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || D < 1) return TM_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return TM_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return TM_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return TM_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return TM_ERR_INVALID_ARG;
  // sizes must stay inside the 32-bit indices used for rows and work items
  const long long rows = static_cast<long long>(B) * N;
  if (rows > (1LL << 31) - 1 || static_cast<long long>(N) * Hq > (1LL << 31) - 1)
    return TM_ERR_INVALID_ARG;
  const long long nqb = (N + TM_BLOCK_M - 1) / TM_BLOCK_M;
  if (nqb * B * Hkv * ((Hq / Hkv + 1) / 2) > (1LL << 31) - 1) return TM_ERR_INVALID_ARG;
  const long long qbytes = rows * Hq * D * 2, kvbytes = rows * Hkv * D * 2;
  if (overlaps(o, qbytes, q, qbytes) || overlaps(o, qbytes, k, kvbytes) ||
      overlaps(o, qbytes, v, kvbytes))
    return TM_ERR_INVALID_ARG;
  return TM_OK;
}

int validate_pattern(int S, int W, int L) {
  if (S < 0 || L < 0 || W < 1) return TM_ERR_INVALID_ARG;
  return TM_OK;
}

// Workspace of the split entry points: NULL with 0 bytes (nothing is split),
// or 16-byte aligned, not overlapping q, k, v or o.
int validate_workspace(const void* q, const void* k, const void* v, const void* o, int B, int Hq,
                       int Hkv, int N, int D, const void* ws, long long ws_bytes) {
  if (ws_bytes < 0 || (!ws && ws_bytes != 0)) return TM_ERR_INVALID_ARG;
  if (!ws) return TM_OK;
  if (!aligned16(ws)) return TM_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * N;
  const long long qbytes = rows * Hq * D * 2, kvbytes = rows * Hkv * D * 2;
  if (overlaps(ws, ws_bytes, q, qbytes) || overlaps(ws, ws_bytes, o, qbytes) ||
      overlaps(ws, ws_bytes, k, kvbytes) || overlaps(ws, ws_bytes, v, kvbytes))
    return TM_ERR_INVALID_ARG;
  return TM_OK;
}

// Scratch of tm_trianglemix_attn_fwd_noalloc: a fixed device array (one per
// device, allocated with the module, never by a call) used as the split
// workspace. Its address is looked up with cudaGetSymbolAddress once per
// device context and cached under that context's unique id: a context that
// is torn down and recreated (cudaDeviceReset) reloads the module, and the
// next call looks the address up again instead of using a stale one.
constexpr long long kScratchBytes = TM_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_split_scratch[kScratchBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct ScratchSlot {
  unsigned long long ctx_id = 0;  // 0: not looked up yet
  void* addr = nullptr;
};
std::mutex g_scratch_mutex;
std::vector<ScratchSlot> g_scratch;  // per device ordinal
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

// Unique id of the calling thread's current context (0 if none is current).
int current_context_id(unsigned long long* id) {
  if (!g_ctx_get_current || !g_ctx_get_id) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || !f1 ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess || !f2)
      return TM_ERR_CUDA;
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return TM_ERR_CUDA;
  *id = 0;
  if (ctx && g_ctx_get_id(ctx, id) != CUDA_SUCCESS) return TM_ERR_CUDA;
  return TM_OK;
}

int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TM_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (static_cast<int>(g_scratch.size()) <= dev) g_scratch.resize(dev + 1);
  ScratchSlot& slot = g_scratch[dev];
  unsigned long long id = 0;
  if (int rc = current_context_id(&id)) return rc;
  if (id == 0 || slot.ctx_id != id) {
    // the lookup also makes the device's primary context current if none is
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_split_scratch) != cudaSuccess || !a) return TM_ERR_CUDA;
    if (int rc = current_context_id(&id)) return rc;
    slot.ctx_id = id;
    slot.addr = a;
  }
  *out = slot.addr;
  return TM_OK;
}

int run(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv, int N, int D,
        float scale, const trimix::Pattern& pat, void* ws, long long ws_bytes, void* stream,
        const int* bs_off = nullptr, const int* bs_idx = nullptr, long long bs_nnz = 0,
        const int* hS = nullptr, const int* hW = nullptr, int inject_cta = -1, int qb_lo = 0,
        int qb_hi = -1) {
  trimix::LaunchArgs a;
  a.qb_lo = qb_lo;
  a.qb_hi = qb_hi;
  a.hS = hS;
  a.hW = hW;
  a.inject_cta = inject_cta;
  a.bs_off = bs_off;
  a.bs_idx = bs_idx;
  a.bs_nnz = bs_nnz;
  a.q = q; a.k = k; a.v = v; a.o = o;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.N = N; a.D = D;
  a.scale = scale;
  a.pat = pat;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  a.stream = stream;
  return trimix::launch_attention(a);
}

// Copy streams and events of the host-buffer layer call, created once per
// device and kept for the life of the process (no device memory). One lock
// per device covers a call's enqueueing, so concurrent calls never interleave
// their event records and waits.
constexpr int kMaxStreamChunks = 64;
constexpr int kDefaultChunkRows = 8192;
struct HostPipe {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, end = nullptr;
  cudaEvent_t loaded[kMaxStreamChunks] = {}, computed[kMaxStreamChunks] = {};
  std::mutex m;
};
constexpr int kMaxPipeDevices = 64;
HostPipe g_pipes[kMaxPipeDevices];
std::mutex g_pipes_mutex;

int host_pipe(HostPipe** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxPipeDevices) return TM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_pipes_mutex);
  HostPipe& hp = g_pipes[dev];
  if (!hp.ready) {
    // create everything, or release what was created and report the failure
    const unsigned ef = cudaEventDisableTiming;
    std::vector<cudaStream_t> streams;
    std::vector<cudaEvent_t> events;
    bool ok = true;
    for (cudaStream_t* st : {&hp.in, &hp.out}) {
      ok = ok && cudaStreamCreateWithFlags(st, cudaStreamNonBlocking) == cudaSuccess;
      if (ok) streams.push_back(*st);
    }
    std::vector<cudaEvent_t*> slots = {&hp.start, &hp.end};
    for (int c = 0; c < kMaxStreamChunks; ++c) {
      slots.push_back(&hp.loaded[c]);
      slots.push_back(&hp.computed[c]);
    }
    for (cudaEvent_t* e : slots) {
      ok = ok && cudaEventCreateWithFlags(e, ef) == cudaSuccess;
      if (ok) events.push_back(*e);
    }
    if (!ok) {
      for (cudaEvent_t e : events) cudaEventDestroy(e);
      for (cudaStream_t st : streams) cudaStreamDestroy(st);
      return TM_ERR_CUDA;
    }
    hp.ready = true;
  }
  *out = &hp;
  return TM_OK;
}

// Rows [r0, r1) of every batch of a [B, N, H, D] bf16 tensor, one copy per batch.
int copy_rows(void* dst, const void* src, int B, int N, int H, int D, int r0, int r1,
              cudaMemcpyKind kind, cudaStream_t st) {
  const size_t row = static_cast<size_t>(H) * D * 2;
  for (int b = 0; b < B; ++b) {
    const size_t off = (static_cast<size_t>(b) * N + r0) * row;
    if (cudaMemcpyAsync(static_cast<char*>(dst) + off, static_cast<const char*>(src) + off,
                        static_cast<size_t>(r1 - r0) * row, kind, st) != cudaSuccess)
      return TM_ERR_CUDA;
  }
  return TM_OK;
}

}  // namespace

extern "C" {

TM_API int tm_causal_attn_fwd_ws(const void* q, const void* k, const void* v, void* o, int B,
                                 int Hq, int Hkv, int N, int D, float scale, void* workspace,
                                 long long workspace_bytes, void* stream) {
  if (int rc = validate_common(q, k, v, o, B, Hq, Hkv, N, D, scale)) return rc;
  if (int rc = validate_workspace(q, k, v, o, B, Hq, Hkv, N, D, workspace, workspace_bytes))
    return rc;
  return run(q, k, v, o, B, Hq, Hkv, N, D, scale, trimix::make_pattern(N, 1, 0, 1, 0), workspace,
             workspace_bytes, stream);
}

TM_API int tm_triangle_attn_fwd_ws(const void* q, const void* k, const void* v, void* o, int B,
                                   int Hq, int Hkv, int N, int D, float scale, int S, int W, int L,
                                   void* workspace, long long workspace_bytes, void* stream) {
  if (int rc = validate_common(q, k, v, o, B, Hq, Hkv, N, D, scale)) return rc;
  if (int rc = validate_pattern(S, W, L)) return rc;
  if (int rc = validate_workspace(q, k, v, o, B, Hq, Hkv, N, D, workspace, workspace_bytes))
    return rc;
  return run(q, k, v, o, B, Hq, Hkv, N, D, scale, trimix::make_pattern(N, 0, S, W, L), workspace,
             workspace_bytes, stream);
}

TM_API int tm_trianglemix_attn_fwd_ws(const void* q, const void* k, const void* v, void* o, int B,
                                      int Hq, int Hkv, int N, int D, float scale, int S, int W,
                                      int L, int layer, int tri_start, void* workspace,
                                      long long workspace_bytes, void* stream) {
  if (layer < 0 || tri_start < 0) return TM_ERR_INVALID_ARG;
  if (layer < tri_start)
    return tm_causal_attn_fwd_ws(q, k, v, o, B, Hq, Hkv, N, D, scale, workspace, workspace_bytes,
                                 stream);
  return tm_triangle_attn_fwd_ws(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L, workspace,
                                 workspace_bytes, stream);
}

TM_API int tm_causal_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int Hq,
                              int Hkv, int N, int D, float scale, void* stream) {
  return tm_causal_attn_fwd_ws(q, k, v, o, B, Hq, Hkv, N, D, scale, nullptr, 0, stream);
}

TM_API int tm_triangle_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int Hq,
                                int Hkv, int N, int D, float scale, int S, int W, int L,
                                void* stream) {
  return tm_triangle_attn_fwd_ws(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L, nullptr, 0, stream);
}

TM_API int tm_trianglemix_attn_fwd(const void* q, const void* k, const void* v, void* o, int B,
                                   int Hq, int Hkv, int N, int D, float scale, int S, int W, int L,
                                   int layer, int tri_start, void* stream) {
  return tm_trianglemix_attn_fwd_ws(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L, layer,
                                    tri_start, nullptr, 0, stream);
}

TM_API int tm_trianglemix_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                                        void* o_host, void* q_dev, void* k_dev, void* v_dev,
                                        void* o_dev, int B, int Hq, int Hkv, int N, int D,
                                        float scale, int S, int W, int L, int layer, int tri_start,
                                        int chunk_rows, void* stream) {
  if (!q_host || !k_host || !v_host || !o_host) return TM_ERR_INVALID_ARG;
  if (int rc = validate_common(q_dev, k_dev, v_dev, o_dev, B, Hq, Hkv, N, D, scale)) return rc;
  if (layer < 0 || tri_start < 0) return TM_ERR_INVALID_ARG;
  const bool causal = layer < tri_start;
  if (!causal)
    if (int rc = validate_pattern(S, W, L)) return rc;
  if (chunk_rows < 0 || chunk_rows % TM_BLOCK_M != 0) return TM_ERR_INVALID_ARG;
  if (chunk_rows == 0) chunk_rows = kDefaultChunkRows;
  // at most kMaxStreamChunks chunks: larger chunks for longer sequences
  const long long min_rows = (static_cast<long long>(N) + kMaxStreamChunks - 1) / kMaxStreamChunks;
  if (chunk_rows < min_rows)
    chunk_rows = static_cast<int>((min_rows + TM_BLOCK_M - 1) / TM_BLOCK_M * TM_BLOCK_M);
  const int n_chunks = static_cast<int>((static_cast<long long>(N) + chunk_rows - 1) / chunk_rows);
  const trimix::Pattern pat =
      causal ? trimix::make_pattern(N, 1, 0, 1, 0) : trimix::make_pattern(N, 0, S, W, L);
  HostPipe* hp = nullptr;
  if (int rc = host_pipe(&hp)) return rc;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(hp->m);
  // the copies start after the work already queued on the caller's stream
  if (cudaEventRecord(hp->start, cs) != cudaSuccess ||
      cudaStreamWaitEvent(hp->in, hp->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp->out, hp->start, 0) != cudaSuccess)
    return TM_ERR_CUDA;
  for (int c = 0; c < n_chunks; ++c) {
    const int r0 = c * chunk_rows;  // < N
    const int r1 = static_cast<int>(std::min<long long>(N, static_cast<long long>(r0) + chunk_rows));
    // chunk c's queries need keys [0, r1) only: its own rows and the chunks before it
    if (int rc = copy_rows(q_dev, q_host, B, N, Hq, D, r0, r1, cudaMemcpyHostToDevice, hp->in))
      return rc;
    if (int rc = copy_rows(k_dev, k_host, B, N, Hkv, D, r0, r1, cudaMemcpyHostToDevice, hp->in))
      return rc;
    if (int rc = copy_rows(v_dev, v_host, B, N, Hkv, D, r0, r1, cudaMemcpyHostToDevice, hp->in))
      return rc;
    if (cudaEventRecord(hp->loaded[c], hp->in) != cudaSuccess ||
        cudaStreamWaitEvent(cs, hp->loaded[c], 0) != cudaSuccess)
      return TM_ERR_CUDA;
    if (int rc = run(q_dev, k_dev, v_dev, o_dev, B, Hq, Hkv, N, D, scale, pat, nullptr, 0, stream,
                     nullptr, nullptr, 0, nullptr, nullptr, -1, r0 / TM_BLOCK_M,
                     (r1 + TM_BLOCK_M - 1) / TM_BLOCK_M))
      return rc;
    if (cudaEventRecord(hp->computed[c], cs) != cudaSuccess ||
        cudaStreamWaitEvent(hp->out, hp->computed[c], 0) != cudaSuccess)
      return TM_ERR_CUDA;
    if (int rc = copy_rows(o_host, o_dev, B, N, Hq, D, r0, r1, cudaMemcpyDeviceToHost, hp->out))
      return rc;
  }
  // the caller's stream completes after the last copy-out
  if (cudaEventRecord(hp->end, hp->out) != cudaSuccess ||
      cudaStreamWaitEvent(cs, hp->end, 0) != cudaSuccess)
    return TM_ERR_CUDA;
  return TM_OK;
}

TM_API int tm_triangle_attn_fwd_heads(const void* q, const void* k, const void* v, void* o, int B,
                                      int Hq, int Hkv, int N, int D, float scale,
                                      const int* S_heads, const int* W_heads, int L,
                                      void* workspace, long long workspace_bytes, void* stream) {
  if (int rc = validate_common(q, k, v, o, B, Hq, Hkv, N, D, scale)) return rc;
  if (!S_heads || !W_heads || L < 0) return TM_ERR_INVALID_ARG;
  if (Hq > 128) return TM_ERR_UNSUPPORTED;
  int S_max = 0, W_max = 1;
  for (int h = 0; h < Hq; ++h) {
    if (S_heads[h] < 0 || W_heads[h] < 1) return TM_ERR_INVALID_ARG;
    S_max = std::max(S_max, S_heads[h]);
    W_max = std::max(W_max, W_heads[h]);
  }
  if (int rc = validate_workspace(q, k, v, o, B, Hq, Hkv, N, D, workspace, workspace_bytes))
    return rc;
  return run(q, k, v, o, B, Hq, Hkv, N, D, scale, trimix::make_pattern(N, 0, S_max, W_max, L),
             workspace, workspace_bytes, stream, nullptr, nullptr, 0, S_heads, W_heads);
}

TM_API int tm_block_sparse_attn_fwd(const void* q, const void* k, const void* v, void* o, int B,
                                    int Hq, int Hkv, int N, int D, float scale,
                                    const int* block_offsets, const int* block_indices,
                                    long long nnz, void* stream) {
  if (int rc = validate_common(q, k, v, o, B, Hq, Hkv, N, D, scale)) return rc;
  if (!block_offsets || nnz < 0 || nnz > (1LL << 31) - 1 || (nnz > 0 && !block_indices))
    return TM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_offsets) & 3u) ||
      (reinterpret_cast<uintptr_t>(block_indices) & 3u))
    return TM_ERR_INVALID_ARG;
  return run(q, k, v, o, B, Hq, Hkv, N, D, scale, trimix::make_pattern(N, 1, 0, 1, 0), nullptr, 0,
             stream, block_offsets, nnz > 0 ? block_indices : block_offsets, nnz);
}

TM_API int tm_trianglemix_sparse_attn_fwd(const void* q, const void* k, const void* v, void* o,
                                          int B, int Hq, int Hkv, int N, int D, float scale,
                                          int S, int W, int L, int layer, int tri_start,
                                          const int* block_offsets, const int* block_indices,
                                          long long nnz, void* stream) {
  if (layer < 0 || tri_start < 0) return TM_ERR_INVALID_ARG;
  if (layer < tri_start)
    return tm_block_sparse_attn_fwd(q, k, v, o, B, Hq, Hkv, N, D, scale, block_offsets,
                                    block_indices, nnz, stream);
  return tm_triangle_attn_fwd(q, k, v, o, B, Hq, Hkv, N, D, scale, S, W, L, stream);
}

namespace {

int validate_discovery(const void* q, const void* k, int B, int Hq, int Hkv, int N, int D,
                       float scale, float alpha, int probes) {
  if (!q || !k || B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv != 0) return TM_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return TM_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k)) return TM_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return TM_ERR_INVALID_ARG;
  if (!std::isfinite(alpha) || alpha < 0.f || alpha > 1.f) return TM_ERR_INVALID_ARG;
  if (probes < 1 || static_cast<long long>(probes) * (Hq / Hkv) > 128) return TM_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * Hkv > 65535) return TM_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * N;
  if (rows > (1LL << 31) - 1 || static_cast<long long>(N) * Hq > (1LL << 31) - 1)
    return TM_ERR_INVALID_ARG;
  return TM_OK;
}

long long max_index_entries(int B, int Hkv, int N) {
  const long long nqb = (N + TM_BLOCK_M - 1) / TM_BLOCK_M;
  return static_cast<long long>(B) * Hkv * nqb * (nqb + 1) / 2;
}

}  // namespace

TM_API int tm_flashprefill_workspace_size(int B, int Hq, int Hkv, int N, int D, int probes,
                                          long long* bytes) {
  if (!bytes) return TM_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv != 0 || probes < 1 ||
      static_cast<long long>(probes) * (Hq / Hkv) > 128)
    return TM_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return TM_ERR_UNSUPPORTED;
  *bytes = trimix::discovery_workspace_bytes(B, Hq, Hkv, N, D, probes);
  return TM_OK;
}

TM_API long long tm_flashprefill_index_capacity(int B, int Hkv, int N) {
  if (B < 1 || Hkv < 1 || N < 1) return -1;
  return max_index_entries(B, Hkv, N);
}

TM_API int tm_flashprefill_block_index(const void* q, const void* k, int B, int Hq, int Hkv, int N,
                                       int D, float scale, float alpha, int probes,
                                       void* workspace, long long workspace_bytes,
                                       int* block_offsets, int* block_indices, long long cap,
                                       float* scores_out, void* stream) {
  if (int rc = validate_discovery(q, k, B, Hq, Hkv, N, D, scale, alpha, probes)) return rc;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || !block_offsets ||
      !block_indices || (reinterpret_cast<uintptr_t>(block_offsets) & 3u) ||
      (reinterpret_cast<uintptr_t>(block_indices) & 3u) ||
      (reinterpret_cast<uintptr_t>(scores_out) & 3u))
    return TM_ERR_INVALID_ARG;
  const long long need = max_index_entries(B, Hkv, N);
  if (cap < need || need > (1LL << 31) - 1) return TM_ERR_INVALID_ARG;
  if (workspace_bytes < trimix::discovery_workspace_bytes(B, Hq, Hkv, N, D, probes))
    return TM_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * N;
  if (overlaps(workspace, workspace_bytes, q, rows * Hq * D * 2) ||
      overlaps(workspace, workspace_bytes, k, rows * Hkv * D * 2))
    return TM_ERR_INVALID_ARG;
  trimix::DiscArgs a;
  a.q = q; a.k = k;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.N = N; a.D = D; a.P = probes;
  a.scale = scale; a.alpha = alpha;
  a.ws = workspace; a.ws_bytes = workspace_bytes;
  a.offsets = block_offsets; a.indices = block_indices;
  a.scores_out = scores_out;
  a.stream = stream;
  return trimix::launch_discovery(a);
}

TM_API int tm_attn_workspace_size(int B, int Hq, int Hkv, int N, int D, int causal, int S, int W,
                                  int L, int num_ctas, long long* bytes) {
  if (!bytes || B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv != 0) return TM_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return TM_ERR_UNSUPPORTED;
  if (!causal && validate_pattern(S, W, L)) return TM_ERR_INVALID_ARG;
  if (static_cast<long long>((N + TM_BLOCK_M - 1) / TM_BLOCK_M) * B * Hkv * ((Hq / Hkv + 1) / 2) >
      (1LL << 31) - 1)
    return TM_ERR_INVALID_ARG;
  return trimix::workspace_bytes(B, Hq, Hkv, N, D, trimix::make_pattern(N, causal, S, W, L),
                                 num_ctas, bytes);
}

TM_API int tm_trianglemix_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                           int B, int Hq, int Hkv, int N, int D, float scale,
                                           int S, int W, int L, int layer, int tri_start,
                                           void* stream) {
  if (layer < 0 || tri_start < 0) return TM_ERR_INVALID_ARG;
  const int causal = layer < tri_start ? 1 : 0;
  if (int rc = validate_common(q, k, v, o, B, Hq, Hkv, N, D, scale)) return rc;
  if (!causal)
    if (int rc = validate_pattern(S, W, L)) return rc;
  const trimix::Pattern pat = causal ? trimix::make_pattern(N, 1, 0, 1, 0)
                                     : trimix::make_pattern(N, 0, S, W, L);
  long long need = 0;
  if (int rc = trimix::workspace_bytes(B, Hq, Hkv, N, D, pat, 0, &need)) return rc;
  // a split larger than the fixed scratch: run the unsplit schedule, which
  // needs no scratch (the same attention; the long items are then not cut)
  if (need == 0 || need > kScratchBytes)
    return run(q, k, v, o, B, Hq, Hkv, N, D, scale, pat, nullptr, 0, stream);
  void* scratch = nullptr;
  if (int rc = scratch_address(&scratch)) return rc;
  return run(q, k, v, o, B, Hq, Hkv, N, D, scale, pat, scratch, kScratchBytes, stream);
}

TM_API long long tm_triangle_kept_pairs(int N, int S, int W, int L) {
  if (N < 1 || validate_pattern(S, W, L)) return -1;
  const trimix::Pattern p = trimix::make_pattern(N, 0, S, W, L);
  long long total = 0;
  for (long long i = 0; i < N; ++i) {
    if (i >= p.N - p.L) {
      total += i + 1;
    } else {
      const long long w = i + 1 < p.W ? i + 1 : p.W;
      long long extra = i + 1 - p.W;
      if (extra > p.S) extra = p.S;
      total += w + (extra > 0 ? extra : 0);
    }
  }
  return total;
}

TM_API long long tm_kept_tiles(int N, int causal, int S, int W, int L) {
  if (N < 1 || (!causal && validate_pattern(S, W, L))) return -1;
  const trimix::Pattern p = trimix::make_pattern(N, causal, S, W, L);
  const int nqb = (N + TM_BLOCK_M - 1) / TM_BLOCK_M;
  long long n = 0;
  for (int qb = 0; qb < nqb; ++qb) n += trimix::block_tiles(p, qb, TM_BLOCK_M, TM_BLOCK_N).count();
  return n;
}

TM_API int tm_tile_list(int N, int causal, int S, int W, int L, int BM, int BN, int* out,
                        long long cap, long long* count) {
  if (N < 1 || BM < 1 || BN < 1 || cap < 0 || !count || (cap > 0 && !out))
    return TM_ERR_INVALID_ARG;
  if (!causal && validate_pattern(S, W, L)) return TM_ERR_INVALID_ARG;
  const trimix::Pattern p = trimix::make_pattern(N, causal, S, W, L);
  const int nqb = (N + BM - 1) / BM;
  long long n = 0;
  for (int qb = 0; qb < nqb; ++qb) {
    const trimix::BlockTiles bt = trimix::block_tiles(p, qb, BM, BN);
    for (int t = 0; t < bt.count(); ++t, ++n) {
      if (n >= cap) continue;
      const int kb = bt.kb(t);
      out[3 * n + 0] = qb;
      out[3 * n + 1] = kb;
      out[3 * n + 2] = trimix::tile_full(p, qb, kb, BM, BN);
    }
  }
  *count = n;
  return TM_OK;
}

TM_API int tm_triangle_tile_list(int N, int S, int W, int L, int BM, int BN, int* out,
                                 long long cap, long long* count) {
  return tm_tile_list(N, 0, S, W, L, BM, BN, out, cap, count);
}

TM_API int tm_debug_dump_tiles(int N, int causal, int S, int W, int L, int* out_dev, long long cap,
                               long long* count, void* stream) {
  if (N < 1 || cap < 0 || !count || (cap > 0 && !out_dev) || !aligned16(out_dev))
    return TM_ERR_INVALID_ARG;
  if (!causal && validate_pattern(S, W, L)) return TM_ERR_INVALID_ARG;
  const long long n = tm_kept_tiles(N, causal, S, W, L);
  if (n < 0) return TM_ERR_INVALID_ARG;
  *count = n;
  return trimix::launch_dump_tiles(trimix::make_pattern(N, causal, S, W, L), out_dev, cap, stream);
}

TM_API int tm_debug_mma_probe(const void* q, const void* k, const void* v, float* s_out,
                              float* o_out, int D, void* stream) {
  if (!q || !k || !v || !s_out || !o_out) return TM_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return TM_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return TM_ERR_UNSUPPORTED;
  return trimix::launch_mma_probe(q, k, v, s_out, o_out, D, stream);
}

TM_API int tm_debug_schedule_window(int B, int Hq, int Hkv, int N, int causal, int S, int W,
                                    int L, int num_ctas, int split, int qb_lo, int qb_hi, int* out,
                                    long long cap, long long* count) {
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv != 0 || num_ctas < 1 || cap < 0 || !count ||
      (cap > 0 && !out))
    return TM_ERR_INVALID_ARG;
  if (!causal && validate_pattern(S, W, L)) return TM_ERR_INVALID_ARG;
  const long long nqb = (N + TM_BLOCK_M - 1) / TM_BLOCK_M;
  if (nqb * B * Hkv * ((Hq / Hkv + 1) / 2) > (1LL << 31) - 1) return TM_ERR_INVALID_ARG;
  if (qb_hi < 0) qb_hi = static_cast<int>(nqb);
  if (qb_lo < 0 || qb_lo >= qb_hi || qb_hi > nqb) return TM_ERR_INVALID_ARG;
  return trimix::debug_schedule(B, Hq, Hkv, N, trimix::make_pattern(N, causal, S, W, L), num_ctas,
                                split, qb_lo, qb_hi, out, cap, count);
}

TM_API int tm_debug_schedule_heads(int B, int Hq, int Hkv, int N, const int* S_heads,
                                   const int* W_heads, int L, int num_ctas, int split, int* out,
                                   long long cap, long long* count) {
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv != 0 || Hq > 128 || num_ctas < 1 ||
      cap < 0 || !count || (cap > 0 && !out) || !S_heads || !W_heads || L < 0)
    return TM_ERR_INVALID_ARG;
  int S_max = 0, W_max = 1;
  for (int h = 0; h < Hq; ++h) {
    if (S_heads[h] < 0 || W_heads[h] < 1) return TM_ERR_INVALID_ARG;
    S_max = std::max(S_max, S_heads[h]);
    W_max = std::max(W_max, W_heads[h]);
  }
  const long long nqb = (N + TM_BLOCK_M - 1) / TM_BLOCK_M;
  if (nqb * B * Hq > (1LL << 31) - 1) return TM_ERR_INVALID_ARG;
  return trimix::debug_schedule(B, Hq, Hkv, N, trimix::make_pattern(N, 0, S_max, W_max, L),
                                num_ctas, (split & 1) | 2, 0, static_cast<int>(nqb), out, cap,
                                count, S_heads, W_heads);
}

TM_API int tm_debug_schedule(int B, int Hq, int Hkv, int N, int causal, int S, int W, int L,
                             int num_ctas, int split, int* out, long long cap, long long* count) {
  return tm_debug_schedule_window(B, Hq, Hkv, N, causal, S, W, L, num_ctas, split, 0, -1, out, cap,
                                  count);
}

TM_API int tm_debug_inject_stall(const void* q, const void* k, const void* v, void* o, int B,
                                 int Hq, int Hkv, int N, int D, float scale, int S, int W, int L,
                                 void* stream) {
  if (int rc = validate_common(q, k, v, o, B, Hq, Hkv, N, D, scale)) return rc;
  if (int rc = validate_pattern(S, W, L)) return rc;
  return run(q, k, v, o, B, Hq, Hkv, N, D, scale, trimix::make_pattern(N, 0, S, W, L), nullptr, 0,
             stream, nullptr, nullptr, 0, nullptr, nullptr, /*inject_cta=*/0);
}

TM_API int tm_get_device_status(void* stream) { return trimix::read_and_clear_device_status(stream); }

TM_API long long tm_debug_launch_count(void) { return trimix::kernel_launches(); }

TM_API const char* tm_status_string(int status) {
  switch (status) {
    case TM_OK: return "ok";
    case TM_ERR_INVALID_ARG: return "invalid argument";
    case TM_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case TM_ERR_CUDA: return "CUDA error";
    case TM_ERR_TIMEOUT: return "kernel gave up on a pipeline wait";
    default: return "unknown status";
  }
}

}  // extern "C"
