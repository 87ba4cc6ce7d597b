// Block pattern discovery for the block-sparse shallow layers, after the
// FlashPrefill summary (section 2.1, instantaneous pattern discovery: uniformly
// spread probe queries against average-pooled key blocks; section 2.2, a
// max-based dynamic threshold instead of a top-k / top-p sort). Included by
// tm_attn.cu inside namespace trimix: it shares that unit's device status word,
// bounded waits and tensor-core helpers.
//
// For batch b, kv head g and q-block I (rows [r0, r1)):
//   pooled keys    kbar_J = mean of k[b, j, g, :] over the keys j of block J
//   probe rows     max(r0, r0 + ((p + 1) (r1 - r0)) / P - 1), p = 0 .. P-1 (the
//                  last one is the block's last row; a block shorter than P
//                  repeats rows), for each q head h of g's group
//   per probe      pi_{h,p}(J) = softmax over J in [0, I] of scale q . kbar_J
//   block score    Score(I, J) = mean over (h, p) of pi_{h,p}(J)
//   kept blocks    J <= I with Score(I, J) >= alpha * max_J' Score(I, J')
// and the kept blocks, ascending, form the CSR index that
// tm_block_sparse_attn_fwd reads. Five launches, all on the caller's stream:
// pool keys and gather probes; scores on the tensor cores (two passes over
// the pooled keys: softmax statistics, then the per-block means); counts;
// an exclusive scan; the index.

constexpr int kDiscThreads = 128;

struct DiscParams {
  int B, Hkv, N, G, nqb, P, R, qbt;  // R = G * P probe rows per q-block; qbt = 128 / R
  float sl2, alpha;                   // scale * log2(e); threshold factor
  const uint16_t* q;                  // bf16 [B, N, Hq, D]
  const uint16_t* k;                  // bf16 [B, N, Hkv, D]
  uint16_t* kbar;                     // bf16 [B * Hkv, nqb, D]
  uint16_t* probes;                   // bf16 [B * Hkv, nqb * R, D]
  float* scores;                      // [B * Hkv, nqb (I), nqb (J)]
  int* counts;                        // [B * Hkv * nqb]
  int* offsets;                       // [B * Hkv * nqb + 1]
  int* indices;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// One CTA per (block J, b * Hkv + g): the pooled key of block J and the probe
// rows of q-block J (q-blocks and key blocks are both 128 rows).
template <int D>
__global__ void __launch_bounds__(kDiscThreads) pool_probe_kernel(const DiscParams p) {
  constexpr int CH = D / 8;              // 16-byte chunks per row
  constexpr int RP = kDiscThreads / CH;  // rows read at once
  __shared__ float red[RP][D];
  const int J = blockIdx.x, bg = blockIdx.y;
  const int b = bg / p.Hkv, g = bg - b * p.Hkv;
  const int t = threadIdx.x, c = t % CH, rp = t / CH;
  const int j0 = J * BN, j1 = imin(p.N, j0 + BN);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int j = j0 + rp; j < j1; j += RP) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(
                              p.k + ((static_cast<size_t>(b) * p.N + j) * p.Hkv + g) * D) + c);
    acc[0] += bf16_lo(w.x); acc[1] += bf16_hi(w.x);
    acc[2] += bf16_lo(w.y); acc[3] += bf16_hi(w.y);
    acc[4] += bf16_lo(w.z); acc[5] += bf16_hi(w.z);
    acc[6] += bf16_lo(w.w); acc[7] += bf16_hi(w.w);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rp][c * 8 + e] = acc[e];
  __syncthreads();
  if (t < D) {
    float s = 0.f;
#pragma unroll
    for (int x = 0; x < RP; ++x) s += red[x][t];
    p.kbar[(static_cast<size_t>(bg) * p.nqb + J) * D + t] =
        __bfloat16_as_ushort(__float2bfloat16_rn(s / static_cast<float>(j1 - j0)));
  }
  const int Hq = p.Hkv * p.G;
  for (int x = t; x < p.R * CH; x += kDiscThreads) {
    const int rr = x / CH, cc = x - rr * CH;
    const int h = rr / p.P, pi = rr - h * p.P;
    const int row = imax(j0, j0 + ((pi + 1) * (j1 - j0)) / p.P - 1);
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(
                              p.q + ((static_cast<size_t>(b) * p.N + row) * Hq + g * p.G + h) * D) +
                          cc);
    reinterpret_cast<uint4*>(p.probes + ((static_cast<size_t>(bg) * p.nqb + J) * p.R + rr) * D)[cc] =
        w;
  }
}

template <int D>
struct DiscCfg {
  static constexpr int kTile = 128 * D * 2;     // 128 probe rows or 128 pooled keys
  static constexpr int kPanel = 128 * 64 * 2;
  static constexpr int kBarOff = 3 * kTile;     // probes, two pooled-key buffers
  static constexpr int kSmem = kBarOff + 64 + 1024;
  static constexpr int kW = kTile / (128 * 4);  // columns per column-sum round (fp32)
};

// One CTA per (qbt consecutive q-blocks, b * Hkv + g): their R-row probe sets
// form one 128-row tile (thread = row = TMEM lane). Pooled-key tiles of 128
// blocks stream through two buffers; a buffer the MMA has finished reading
// doubles as the column-sum scratch of that tile.
template <int D>
__global__ void __launch_bounds__(kDiscThreads, 2)
    score_kernel(const __grid_constant__ CUtensorMap tp, const __grid_constant__ CUtensorMap tkb,
                 const __grid_constant__ DiscParams p) {
  using C = DiscCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);  // probes, kbar x2, mma
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  int* abort_flag = reinterpret_cast<int*>(bars + 5);
  const int t = threadIdx.x, warp = t >> 5;
  const int bg = blockIdx.y, I0 = blockIdx.x * p.qbt;
  const int I_last = imin(p.nqb, I0 + p.qbt) - 1;
  const int nkt = I_last / BN + 1;  // pooled-key tiles covering J <= I_last
  const int total = 2 * nkt;        // pass 0: softmax statistics; pass 1: block means
  if (t == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sp = smem_addr(smem), sk = sp + C::kTile;
  if (t == 0) {
    tma_prefetch_desc(&tp);
    tma_prefetch_desc(&tkb);
    mbar_arrive_expect_tx(&bars[0], C::kTile);
    for (int pn = 0; pn < D / 64; ++pn)
      tma_load_3d(sp + pn * C::kPanel, &tp, &bars[0], pn * 64, I0 * p.R, bg);
    mbar_arrive_expect_tx(&bars[1], C::kTile);
    for (int pn = 0; pn < D / 64; ++pn)
      tma_load_3d(sk + pn * C::kPanel, &tkb, &bars[1], pn * 64, 0, bg);
  }
  const int qi = t / p.R;
  const int I = I0 + qi;
  const bool valid = qi < p.qbt && I < p.nqb;
  const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
  float m = -INFINITY, z = 0.f;
  // thread 0's record of what it put in flight and saw land (for a clean abort)
  int issued[2] = {1, 0}, landed[2] = {0, 0}, mma_issued = 0, mma_done = 0;
  bool ok = wait_bar(&bars[0], 0, abort_flag, kSiteDisc);
  const bool probes_landed = ok;
  int it = 0;
  for (; it < total; ++it) {
    const int pass = it >= nkt ? 1 : 0, kt = pass ? it - nkt : it, buf = it & 1;
    if (t == 0 && it + 1 < total) {  // the other buffer is free since the last barrier
      const int nk = it + 1 >= nkt ? it + 1 - nkt : it + 1;
      fence_proxy_async_smem();        // column sums written there before the async copy
      mbar_arrive_expect_tx(&bars[1 + (buf ^ 1)], C::kTile);
      for (int pn = 0; pn < D / 64; ++pn)
        tma_load_3d(sk + (buf ^ 1) * C::kTile + pn * C::kPanel, &tkb, &bars[1 + (buf ^ 1)],
                    pn * 64, nk * BN, bg);
      ++issued[buf ^ 1];
    }
    ok = ok && wait_bar(&bars[1 + buf], (it >> 1) & 1, abort_flag, kSiteDisc);
    if (ok) ++landed[buf];
    if (t == 0 && ok) {
      tc_fence_after();
      issue_qk<D>(tmem, desc_lo_sw128(sp, 16), desc_lo_sw128(sk + buf * C::kTile, 16));
      mma_commit(&bars[3]);
      ++mma_issued;
    }
    ok = ok && wait_bar(&bars[3], it & 1, abort_flag, kSiteDisc);
    if (ok) ++mma_done;
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
    uint32_t sr[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_addr + 32 * c, sr[c]);
    tmem_wait_ld(sr[0]);
    reg_fence(sr[1]);
    reg_fence(sr[2]);
    reg_fence(sr[3]);
    tc_fence_before();
    const int J0 = kt * BN;
    const int n_keep = valid ? imin(BN, I - J0 + 1) : 0;  // columns J0 .. I of this tile
    if (pass == 0) {
      if (n_keep > 0) {
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int x = 0; x < 32; ++x)
            if (32 * c + x < n_keep) mx = fmaxf(mx, __uint_as_float(sr[c][x]) * p.sl2);
        const float m_new = fmaxf(m, mx);
        float zs = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int x = 0; x < 32; ++x)
            if (32 * c + x < n_keep) zs += ex2(__uint_as_float(sr[c][x]) * p.sl2 - m_new);
        z = z * ex2(m - m_new) + zs;  // ex2(-inf) = 0 on the first tile
        m = m_new;
      }
    } else {
      float* cs = reinterpret_cast<float*>(smem + C::kTile + buf * C::kTile);
      constexpr int W = C::kW;
      const float inv = (n_keep > 0 && z > 0.f) ? 1.f / z : 0.f;
#pragma unroll
      for (int h = 0; h < 128 / W; ++h) {
        // this row's probabilities of columns [h W, h W + W), rotated by the row
        // number so that neither the row-wise writes nor the column-wise
        // reads collide in a shared-memory bank
#pragma unroll
        for (int x = 0; x < W; ++x) {
          const int col = h * W + x;
          const float sv = __uint_as_float(sr[col >> 5][col & 31]);
          cs[t * W + ((x + t) & (W - 1))] = col < n_keep ? ex2(sv * p.sl2 - m) * inv : 0.f;
        }
        __syncthreads();
        const int x = t & (W - 1);
        for (int q2 = t / W; q2 < p.qbt && I0 + q2 < p.nqb; q2 += 128 / W) {
          float s = 0.f;
          for (int rr = q2 * p.R; rr < q2 * p.R + p.R; ++rr) s += cs[rr * W + ((x + rr) & (W - 1))];
          const int J = J0 + h * W + x;
          if (J < p.nqb)
            p.scores[(static_cast<size_t>(bg) * p.nqb + I0 + q2) * p.nqb + J] =
                s / static_cast<float>(p.R);
        }
        // generic writes to this buffer, ordered before the next async copy into it
        fence_proxy_async_smem();
        __syncthreads();
      }
    }
    __syncthreads();
  }
  if (it < total && t == 0) {  // gave up: let the copies and the MMA in flight land first
    if (!probes_landed) drain_wait(&bars[0], 0);
    for (int b2 = 0; b2 < 2; ++b2)
      if (issued[b2] > landed[b2]) drain_wait(&bars[1 + b2], landed[b2] & 1);
    if (mma_issued > mma_done) drain_wait(&bars[3], mma_done & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// One warp per list (b * Hkv + g, I): the kept count under the threshold.
__global__ void count_kernel(const DiscParams p) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (wid >= p.B * p.Hkv * p.nqb) return;
  const int I = wid % p.nqb;
  const float* row = p.scores + static_cast<size_t>(wid) * p.nqb;
  float mx = 0.f;
  for (int J = lane; J <= I; J += 32) mx = fmaxf(mx, row[J]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float th = p.alpha * mx;
  int cnt = 0;
  for (int J = lane; J <= I; J += 32) cnt += row[J] >= th ? 1 : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) p.counts[wid] = cnt;
}

// Exclusive scan of the counts into the offsets (one CTA of 1024 threads).
__global__ void __launch_bounds__(1024) scan_kernel(const DiscParams p) {
  __shared__ int part[1024];
  const int n = p.B * p.Hkv * p.nqb, t = threadIdx.x;
  const int per = (n + 1023) / 1024, a = imin(n, t * per), e = imin(n, a + per);
  int s = 0;
  for (int i = a; i < e; ++i) s += p.counts[i];
  part[t] = s;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const int v = t >= off ? part[t - off] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  int base = t ? part[t - 1] : 0;
  for (int i = a; i < e; ++i) {
    p.offsets[i] = base;
    base += p.counts[i];
  }
  if (t == 1023) p.offsets[n] = part[1023];
}

// One warp per list: the kept blocks in ascending order (the same comparisons
// as count_kernel, so each list fills exactly its counted slots).
__global__ void write_index_kernel(const DiscParams p) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (wid >= p.B * p.Hkv * p.nqb) return;
  const int I = wid % p.nqb;
  const float* row = p.scores + static_cast<size_t>(wid) * p.nqb;
  float mx = 0.f;
  for (int J = lane; J <= I; J += 32) mx = fmaxf(mx, row[J]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float th = p.alpha * mx;
  int pos = p.offsets[wid];
  for (int J0 = 0; J0 <= I; J0 += 32) {
    const int J = J0 + lane;
    const bool keep = J <= I && row[J] >= th;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) p.indices[pos + __popc(bal & ((1u << lane) - 1u))] = J;
    pos += __popc(bal);
  }
}
