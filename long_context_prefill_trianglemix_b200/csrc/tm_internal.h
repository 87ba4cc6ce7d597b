// Internal interface between the C ABI (tm_api.cu) and the kernel translation
// unit (tm_attn.cu). Not installed; not part of the public ABI.
#pragma once

#include <cstdint>

#include "tm_tiles.cuh"

namespace trimix {

// Codes the kernels write into the device status word.
enum DeviceStatus : int { kDevOk = 0, kDevTimeout = 1 };

struct LaunchArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  int B, Hq, Hkv, N, D;
  float scale;
  Pattern pat;
  void* ws;           // split workspace (device), or nullptr: no item is split
  long long ws_bytes;
  const int* bs_off;  // block-sparse index (device CSR), or nullptr: pat's tile list
  const int* bs_idx;
  long long bs_nnz;
  const int* hS;      // per-head sinks and windows (host, Hq each), or nullptr
  const int* hW;
  int inject_cta;     // test hook: -1, or the CTA whose first Q is never delivered
  void* stream;
  int qb_lo = 0;      // the q-blocks [qb_lo, qb_hi) of the sequence; qb_hi -1: to the end
  int qb_hi = -1;
};

struct DiscArgs {
  const void* q;
  const void* k;
  int B, Hq, Hkv, N, D, P;
  float scale, alpha;
  void* ws;
  long long ws_bytes;
  int* offsets;
  int* indices;
  float* scores_out;  // optional: the block scores land here instead of the workspace
  void* stream;
};

// All return a tm_status value.
int launch_attention(const LaunchArgs& a);
int launch_dump_tiles(const Pattern& p, int* out_dev, long long cap, void* stream);
int launch_mma_probe(const void* q, const void* k, const void* v, float* s_out, float* o_out,
                     int D, void* stream);
int read_and_clear_device_status(void* stream);
// Kernels launched by the library so far in this process.
long long kernel_launches();
int launch_discovery(const DiscArgs& a);
long long discovery_workspace_bytes(int B, int Hq, int Hkv, int N, int D, int P);
int debug_schedule(int B, int Hq, int Hkv, int N, const Pattern& pat, int max_ctas, int split,
                   int qb_lo, int qb_hi, int* out, long long cap, long long* count,
                   const int* hS = nullptr, const int* hW = nullptr);
// Workspace bytes the split schedule needs on num_ctas CTAs (<= 0: the
// current device's SM count); 0 if no item is split.
int workspace_bytes(int B, int Hq, int Hkv, int N, int D, const Pattern& pat, int num_ctas,
                    long long* bytes);

}  // namespace trimix
