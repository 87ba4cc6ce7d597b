// TriangleMix prefill attention for sm_100a: one persistent, warp-specialised
// kernel template for the dense causal pattern and the static triangle pattern.
//
// What is computed is exact masked softmax attention over the kept key set of
// each query row (TriangleMix blog post, sections 介绍 and 缘由; 36kr interview,
// lead paragraphs): the triangle keeps the first S sink keys, the W most recent
// keys and, for the last L query rows, every causal key.
//
// CTA layout (384 threads, one CTA per SM, persistent):
//   warps 0-3  softmax warpgroup 0: rows of Q tile 0 (TMEM lanes 0..127)
//   warps 4-7  softmax warpgroup 1: rows of Q tile 1
//   warp  8    TMA producer (one elected thread): Q tiles, then K/V tiles
//   warp  9    tcgen05 issuer (the warp in step, one elected lane issues) and TMEM owner
//   warps 10-11 idle (they complete the third warpgroup for setmaxnreg)
// The kernel is launched at 168 registers per thread (384 x 168 = 64512);
// the third warpgroup drops to 88 and the softmax warpgroups rise to 208
// (2 x 128 x 208 + 128 x 88 = 64512), so the row of 128 scores stays in
// registers. The host refuses to launch a build whose register count differs.
// A work item is (batch, kv head, pair of q heads of that kv head's group,
// q-block), or, in per-head band launches and causal launches of odd group
// sizes, two consecutive q-blocks of one q head: both Q tiles read the same
// K/V stream, which is loaded once. Only the kept k-blocks are visited
// (tm_tiles.cuh); elementwise masking runs only on the tiles that need it.
//
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
// The output leaves through shared memory and TMA stores (one 4 KB slot per
// softmax warp), so the epilogue does not flood the load/store path with
// scattered 16-byte global writes while the other warpgroup is still working.
// P (bf16) overwrites the first 64 columns of its S tile once S has been read
// into registers, and feeds the P.V MMA directly from TMEM.
//
// MMA issue order per item (K_t, V_t are ring slots, in load order):
//   S0=Q0.K0  S1=Q1.K0 | for t: O0+=P0.V_t  S0=Q0.K_{t+1}  O1+=P1.V_t  S1=Q1.K_{t+1}
// so one softmax warpgroup works while the tensor core runs the other's MMAs.
//
// Every wait is bounded (about two seconds). On expiry the kernel records a
// timeout in g_status, every role leaves its loop, in-flight copies and MMAs
// are drained with bounded waits, TMEM is freed and the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <mutex>
#include <vector>

#include "tm.h"
#include "tm_internal.h"
#include "tm_sm100.cuh"
#include "tm_tiles.cuh"

namespace trimix {

using namespace sm100;

__device__ int g_status = 0;
__device__ int g_status_where = 0;

constexpr int BM = TM_BLOCK_M;
constexpr int BN = TM_BLOCK_N;
static_assert(BM == 128 && BN == 128, "tile shape is fixed by the TMEM layout");
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 208;
constexpr int kSideRegs = 88;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kSideRegs == kThreads * kLaunchRegs,
              "register split must use exactly the registers the CTA is launched with");
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kMaxCtas = 192;
constexpr int kMaxBandHeads = 128;  // q heads of a per-head band launch
constexpr uint32_t kTmemCols = 512;
// Lazy running max (log2 domain): it moves only when a tile's max exceeds it
// by more than kRescaleThreshold, and then to that max plus kRescaleMargin, so
// the O rescale (a TMEM round trip of all of O on the softmax's critical path,
// about a thousand cycles) stays rare even when scores vary widely, as they do
// with outlier channels in q and k. Weights stay below 2^48: P is bf16 and O,
// l are fp32, whose exponent range leaves O = sum p.v finite for |v| up to
// about 2^62 over 2^17 keys; each new reference leaves the weights at most
// 2^-8 below their exact values' scale, and both bf16 and fp32 round relative
// to the value, so the weights' accuracy does not depend on the reference.
constexpr float kRescaleThreshold = 48.0f;
constexpr float kRescaleMargin = 8.0f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
#ifndef TM_POLY_PAIRS
#define TM_POLY_PAIRS 0
#endif
// Of every 32 pairs of probabilities, this many are exponentiated on the FMA
// pipe (ex2_poly) and the rest on MUFU, to balance the two units.
constexpr int kPolyPairs = TM_POLY_PAIRS;
static_assert(kPolyPairs >= 0 && kPolyPairs <= 32, "pairs per 32");
// Per-item fixed cost (Q load, first S, last P.V, epilogue) in units of one
// visited tile, used only to balance the persistent work split.
constexpr long long kItemOverheadTiles = 3;
constexpr uint64_t kDrainLimitNs = 100000000ull;
// Cutting heavy items (split schedules): a piece costs at most this fraction
// of a CTA's share, holds at least kMinPieceTiles tiles, an item is cut into
// at most kMaxSplit pieces, and writing a partial costs about one tile.
constexpr double kSplitShare = 0.5;
constexpr int kMinPieceTiles = 8;
constexpr int kMaxSplit = 16;
constexpr long long kSplitOverheadTiles = 1;

// Where a wait gave up (recorded with the timeout, for diagnosis).
enum WaitSite : int {
  kSiteQEmpty = 1, kSiteKvEmpty, kSiteQFull, kSiteKvFull, kSiteOEmpty, kSitePFull,
  kSiteSFull, kSiteOFull, kSiteProbe, kSiteDisc, kSiteDescEmpty, kSiteDescFull
};

template <int D>
struct Cfg {
  static constexpr int kTileBytes = BM * D * 2;  // one Q, K or V tile (BM == BN)
  static constexpr int kPanelBytes = BM * 64 * 2; // one 128-byte-wide swizzle panel
  static constexpr int kPanels = D / 64;
  static constexpr int kStages = (D == 128) ? 4 : 8;
  static constexpr int kRingOff = 2 * kTileBytes;
  // Output staging: one 4 KB slot per softmax warp (32 rows x 64 bf16 columns,
  // 128-byte swizzled), written from registers and sent out by a TMA store.
  static constexpr int kStageOff = kRingOff + kStages * kTileBytes;
  static constexpr int kStageSlotBytes = 32 * 128;
  static constexpr int kBarOff = kStageOff + 8 * kStageSlotBytes;
  static constexpr int kSmemBytes = kBarOff + 768 + 1024;  // barriers + alignment slack
  static constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128;
  static constexpr uint32_t kTmemO0 = 256, kTmemO1 = 256 + D;
  static constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, 0, 0);  // Q, K both K-major
  static constexpr uint32_t kIdescO = idesc_bf16_f32(BM, D, 0, 1);   // V is MN-major
};

// What the producer tells the softmax warpgroups about each item, through a
// ring of kDescRing slots in shared memory (qb < 0 ends the CTA's work).
struct ItemDesc {
  int b, g, qb, h0, h1, v1, t0, t1, split, hunit, pad0, pad1;
};
constexpr int kDescRing = 4;

template <int NST>
struct Bars {
  uint64_t q_full, q_empty;
  uint64_t kv_full[NST], kv_empty[NST];
  uint64_t s_full[2], p_full[4], o_full[2], o_empty[2];  // p_full[2w + h]: half h of P_w
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  // The producer's item descriptor for the MMA issuer: visited tiles (0 ends
  // the CTA's work) and whether a second Q tile is present. Written before the
  // producer's arrival on q_full, read after the issuer's wait on it.
  int item_T, item_v1;
  uint64_t desc_full[kDescRing], desc_empty[kDescRing];
  ItemDesc desc[kDescRing];
};
static_assert(sizeof(Bars<8>) <= 768 && sizeof(Bars<4>) <= 768, "barrier block is 768 bytes");

struct AttnParams {
  // nqb q-blocks of work, qb0 .. qb0 + nqb - 1 (a window of the nqb_all
  // q-blocks of the sequence; the whole sequence unless the caller streams
  // it in row chunks); q-block indices in items are global.
  int B, Hq, Hkv, N, G, npairs, nqb, units, qb0, nqb_all;
  Pattern pat;
  float sl2;  // softmax scale * log2(e)
  // Items run q-block major (longest q-blocks first), the (batch, kv head,
  // pair) units inside. The n_hqb heaviest q-blocks (the last-L blocks of the
  // triangle) give n_hunits = n_hqb * units heavy items; those of the first
  // n_sqb q-blocks are each cut into nsplit pieces of their tile list. The
  // n_big big pieces (n_sbig = n_sqb * units * nsplit pieces of cut items,
  // then the other heavy items whole) are dealt round-robin: CTA c takes c,
  // c + grid, ... Every other item is dealt in
  // strided rounds, so that the CTAs running at the same time work on
  // neighbouring q-blocks of every kv head and each K/V tile is read from DRAM
  // about once per round. The first n_a CTAs hold one piece more than the rest
  // and join the rounds n_skip rounds late. Normal item j of CTA c (j counted
  // from 0, item index n_hunits + that):
  //   c >= n_a and j < n_skip:  (c - n_a) + j * (grid - n_a)
  //   otherwise:                 n_skip * (grid - n_a) + (j - s_c) * grid + c,
  //                              s_c = n_skip if c >= n_a else 0
  int n_hqb, n_hunits, n_sqb, n_sbig, n_big, n_a, n_skip;
  // With an odd group size one pair per kv head holds a single Q tile. The
  // pair of an item is rotated by pair_rot per q-block slot (pair digit + qi *
  // pair_rot, mod npairs), chosen so that the pair a CTA gets changes through
  // all npairs values along its stride and every CTA gets its share of the
  // cheap single-tile items (0 for even group sizes). The rotation permutes
  // the pairs inside each (kv head, q-block) group, whose items stay adjacent.
  // kv_rot rotates the kv head the same way (per-head band launches, whose kv
  // heads differ in cost); it permutes whole groups, which stay adjacent too.
  int pair_rot, kv_rot;
  // Chunked group order of the normal items (gchunk != 0; causal launches of
  // even group sizes): the normal q-blocks are cut, from the longest, into
  // chunks of qchunk q-blocks; chunk by chunk, every (batch, kv head) takes
  // its turn with the chunk's q-blocks (longest first, pairs fastest). With
  // qchunk = grid / npairs each turn is one strided round, so the CTAs running
  // at the same time read the K/V of a single kv head, which stays in L2 for
  // the whole round however far the CTAs drift apart along their tile lists;
  // consecutive turns have the same cost profile, which the reversed odd
  // rounds balance. The q-blocks left after the last full chunk (the
  // shortest; their K/V fits in L2 for all heads) run q-block major.
  int gchunk, qchunk;
  // Test hook (-1 in every product launch): the producer of this CTA delivers
  // no Q for its first item and leaves, so the issuer's bounded wait on q_full
  // runs out; the CTA records a timeout and every role exits cleanly.
  int inject_cta;
  // Split pieces (nsplit > 1): each writes its unnormalised partial (O, running
  // max m, sum l) of every 32-row warp slice to ws_rec and counts itself in
  // ws_cnt (one counter per cut item, Q tile and warp, zero at launch); the
  // piece that arrives last merges all partials in split order.
  int nsplit;
  float* ws_rec;
  int* ws_cnt;
  // Block-sparse launches (bs_off != nullptr): the tile list of item (b, kv
  // head g, q-block qb) is bs_idx[bs_off[r] .. bs_off[r + 1]), r = (b * Hkv +
  // g) * nqb_all + qb, offsets clamped to [0, bs_nnz]; pat is the causal pattern.
  const int* bs_off;
  const int* bs_idx;
  int bs_nnz;
  // Per-head bands (ph != 0): q head h keeps the sinks [0, hS[h]) and a window
  // of hW[h] positions (L and the rest of pat shared; pat.S, pat.W hold the
  // maxima). The heads of each kv group are paired in the order hperm (sorted
  // by band on the host, so the two heads of a pair have similar bands); an
  // item visits the union of its two heads' tile lists, which is the closed
  // form at (max S, max W) since both kept sets are [0, S) U [i - W + 1, i].
  int ph;
  // Q-block pairs (qpair != 0): the two Q tiles of an item are consecutive
  // q-blocks qb, qb + 1 of one q head instead of two heads of a group. Per-head
  // band launches use them because heads of one group can have very different
  // bands, while the union of two neighbouring q-blocks' lists wastes about one
  // tile per Q tile. Causal launches with an odd group size use them because a
  // head pair would leave one head of every group alone in an item, with one
  // softmax warpgroup idle; for causal rows the union is the later q-block's
  // list, one tile more than the earlier one's. The schedule's q-block x is
  // then the pair of q-blocks 2x - qdelta, 2x + 1 - qdelta (qdelta puts the
  // first full-causal q-block of the last-L rows at the start of a pair, and
  // for causal launches leaves q-block 0 alone when the count is odd); a pair
  // cut by the sequence's ends holds one Q tile.
  int qpair, qdelta;
  int hS[kMaxBandHeads], hW[kMaxBandHeads];
  unsigned char hperm[kMaxBandHeads];
};

__host__ __device__ __forceinline__ int big_count(const AttnParams& p, int c, int g) {
  return c < p.n_big ? (p.n_big - c + g - 1) / g : 0;
}

// Normal index (counted from 0 after the big items) of CTA c's j-th normal item.
__host__ __device__ __forceinline__ long long normal_index(const AttnParams& p, int c, int g, int j) {
  const int ga = g - p.n_a;
  if (c >= p.n_a && j < p.n_skip)
    return static_cast<long long>(c - p.n_a) + static_cast<long long>(j) * ga;
  // main rounds r = 0, 1, ...: odd rounds are dealt in reverse CTA order, so a
  // CTA that drew a long item of its round draws a short one next and the
  // CTAs' positions in the tile streams do not drift apart
  const int r = c >= p.n_a ? j - p.n_skip : j;
  return static_cast<long long>(p.n_skip) * ga + static_cast<long long>(r) * g +
         ((r & 1) ? g - 1 - c : c);
}

__host__ __device__ __forceinline__ int work_count(const AttnParams& p, int c, int g) {
  const long long n_norm = static_cast<long long>(p.nqb) * p.units - p.n_hunits;
  // largest j with normal_index(j) < n_norm, + 1 (monotone in j)
  int lo = 0, hi = static_cast<int>(n_norm) + 1;
  while (lo < hi) {
    const int mid = (lo + hi) / 2;
    if (normal_index(p, c, g, mid) < n_norm) lo = mid + 1; else hi = mid;
  }
  return big_count(p, c, g) + lo;
}

__host__ __device__ __forceinline__ int work_item(const AttnParams& p, int c, int g, int k) {
  const int nb = big_count(p, c, g);
  return k < nb ? c + k * g : p.n_big + static_cast<int>(normal_index(p, c, g, k - nb));
}

// One unit of work: Q tiles of q heads h0 (and h1 if v1) of q-block qb, kv
// head g of batch b, over tiles [t0, min(t1, count)) of the q-block's tile
// list. split >= 0 marks a piece of a heavy item (hunit: its index among the
// heavy items).
struct Item {
  int b, g, qb, h0, h1, v1;
  int t0, t1, split, hunit;
};

constexpr int kAllTiles = 0x7fffffff;

// The q heads of pair pr of kv head g (h1 = h0 when the group ends in a single head).
__host__ __device__ __forceinline__ void pair_heads(const AttnParams& p, int g, int pr, Item& it) {
  const int hp = g * p.G + 2 * pr;
  it.v1 = (2 * pr + 1 < p.G) ? 1 : 0;
  it.h0 = p.ph ? p.hperm[hp] : hp;
  it.h1 = it.v1 ? (p.ph ? p.hperm[hp + 1] : hp + 1) : it.h0;
}

// The Q tiles of unit digit pr of kv head g at schedule q-block x: head pair pr
// of q-block x, or with q-block pairs the q-blocks 2x - qdelta, 2x + 1 - qdelta
// of head pr.
__host__ __device__ __forceinline__ void unit_tiles(const AttnParams& p, int x, int g, int pr,
                                                    Item& it) {
  if (p.qpair) {
    const int qa = 2 * x - p.qdelta;
    it.qb = imax(qa, 0);
    it.v1 = (qa >= 0 && qa + 1 < p.nqb_all) ? 1 : 0;
    it.h0 = it.h1 = g * p.G + pr;
  } else {
    it.qb = x;
    pair_heads(p, g, pr, it);
  }
}

// Pattern of one q head, and of an item (the union of its heads' patterns).
__host__ __device__ __forceinline__ Pattern head_pattern(const AttnParams& p, int h) {
  Pattern q = p.pat;
  if (p.ph) {
    q.S = p.hS[h];
    q.W = p.hW[h];
  }
  return q;
}
__host__ __device__ __forceinline__ Pattern item_pattern(const AttnParams& p, const Item& it) {
  Pattern q = p.pat;
  if (p.ph && !p.qpair) {
    q.S = imax(p.hS[it.h0], p.hS[it.h1]);
    q.W = imax(p.hW[it.h0], p.hW[it.h1]);
  } else if (p.ph) {
    q.S = p.hS[it.h0];
    q.W = p.hW[it.h0];
  }
  return q;
}

// Rows of schedule q-block x: [r0, r1] (two q-blocks with q-block pairs), and
// the tile list of an item (the union of its Q tiles' lists).
__host__ __device__ __forceinline__ BlockTiles sched_tiles(const AttnParams& p, const Pattern& pat,
                                                           int x) {
  if (!p.qpair) return block_tiles(pat, x, BM, BN);
  const int qa = 2 * x - p.qdelta;
  const int r0 = imax(qa, 0) * BM;
  return block_tiles_rows(pat, r0, imin(p.N, (qa + 2) * BM) - 1, BN);
}
__host__ __device__ __forceinline__ BlockTiles item_tiles(const AttnParams& p, const Item& it) {
  if (!p.qpair) return block_tiles(item_pattern(p, it), it.qb, BM, BN);
  return block_tiles_rows(item_pattern(p, it), it.qb * BM,
                          imin(p.N, (it.qb + 1 + it.v1) * BM) - 1, BN);
}

__host__ __device__ __forceinline__ Item decode_item(const AttnParams& p, int item) {
  Item it;
  const int qi = item / p.units;
  const int u = item - qi * p.units;
  const int x = p.qb0 + p.nqb - 1 - qi;  // longest q-blocks first
  // unit digits, fastest first: pair, kv head, batch. The pairs of one kv head
  // and q-block are consecutive items, which the strided rounds hand to
  // neighbouring CTAs: they walk the same tile list in lockstep, so each K/V
  // tile is fetched from DRAM once for all of them.
  const int pr = (u % p.npairs + static_cast<int>(static_cast<long long>(qi) * p.pair_rot % p.npairs)) %
                 p.npairs;
  const int gb = u / p.npairs;
  it.g = (gb % p.Hkv + static_cast<int>(static_cast<long long>(qi) * p.kv_rot % p.Hkv)) % p.Hkv;
  it.b = gb / p.Hkv;
  unit_tiles(p, x, it.g, pr, it);
  it.t0 = 0;
  it.t1 = kAllTiles;
  it.split = -1;
  it.hunit = -1;
  return it;
}

// Big piece bi < n_sbig: cut q-block slot qi, then split s, then unit u (so
// CTAs running at the same time read the same tile range of a kv head); the
// rest are whole heavy items in item order.
__host__ __device__ __forceinline__ Item decode_piece(const AttnParams& p, int bi) {
  if (bi >= p.n_sbig) return decode_item(p, p.n_sqb * p.units + (bi - p.n_sbig));
  const int per_q = p.units * p.nsplit;
  const int qi = bi / per_q;
  const int rem = bi - qi * per_q;
  const int s = rem / p.units;
  const int u = rem - s * p.units;
  Item it = decode_item(p, qi * p.units + u);
  if (p.nsplit > 1) {
    const int T = item_tiles(p, it).count();
    it.t0 = static_cast<int>(static_cast<long long>(T) * s / p.nsplit);
    it.t1 = static_cast<int>(static_cast<long long>(T) * (s + 1) / p.nsplit);
    it.split = s;
    it.hunit = qi * p.units + u;
  }
  return it;
}

// The tile list of one item: the closed form of the pattern, or a run of the
// caller's block index. Index entries are clamped to [-1, nqb]: TMA reads
// zeros outside the tensor, and the softmax masks such tiles completely, so a
// malformed index gives masked tiles, never an access outside q, k or v.
struct TileSrc {
  BlockTiles bt;
  const int* idx;  // nullptr: closed form
  int n, nkb;
  __device__ __forceinline__ int count() const { return idx ? n : bt.count(); }
  __device__ __forceinline__ int kb(int t) const {
    if (!idx) return bt.kb(t);
    const int v = __ldg(idx + t);
    return v < -1 ? -1 : (v > nkb ? nkb : v);
  }
};

__device__ __forceinline__ TileSrc tile_src(const AttnParams& p, const Item& it) {
  TileSrc s;
  s.idx = nullptr;
  s.n = 0;
  s.nkb = p.nqb_all;
  if (p.bs_off) {
    const long long r = (static_cast<long long>(it.b) * p.Hkv + it.g) * p.nqb_all + it.qb;
    const int o0 = imin(imax(__ldg(p.bs_off + r), 0), p.bs_nnz);
    const int o1 = imin(imax(__ldg(p.bs_off + r + 1), o0), p.bs_nnz);
    s.idx = p.bs_idx + o0;
    s.n = o1 - o0;
    s.bt.n_a = s.bt.b_lo = s.bt.n_b = 0;
  } else {
    s.bt = item_tiles(p, it);
  }
  return s;
}

// Normal item n (counted from 0 after the big items) in the launch's order.
__host__ __device__ __forceinline__ Item normal_item(const AttnParams& p, long long n) {
  const long long per_full = static_cast<long long>(p.qchunk) * p.units;
  const long long n_chunked = (p.nqb - p.n_hqb) / p.qchunk * per_full;
  // q-block major: every item without the chunked order, and the q-blocks
  // after the last full chunk (the shortest ones) with it
  if (!p.gchunk || n >= n_chunked) return decode_item(p, static_cast<int>(p.n_hunits + n));
  const int k = static_cast<int>(n / per_full);      // chunk
  const int rem = static_cast<int>(n - k * per_full);
  const int per_gb = p.qchunk * p.npairs;
  const int gb = rem / per_gb;
  const int r2 = rem - gb * per_gb;
  const int qi = p.n_hqb + k * p.qchunk + r2 / p.npairs;
  Item it;
  it.g = gb % p.Hkv;
  it.b = gb / p.Hkv;
  unit_tiles(p, p.qb0 + p.nqb - 1 - qi, it.g, r2 % p.npairs, it);
  it.t0 = 0;
  it.t1 = kAllTiles;
  it.split = -1;
  it.hunit = -1;
  return it;
}

// Item k of CTA c's work (big pieces first, then its normal items).
__host__ __device__ __forceinline__ Item work_item_at(const AttnParams& p, int c, int g, int k) {
  const int nb = big_count(p, c, g);
  return k < nb ? decode_piece(p, c + k * g) : normal_item(p, normal_index(p, c, g, k - nb));
}

__device__ __forceinline__ void record_timeout(int site) {
  if (atomicCAS(&g_status, kDevOk, kDevTimeout) == kDevOk) g_status_where = site;
}

// Bounded mbarrier wait. false = gave up (timeout here, or abort seen).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                      int site) {
  const uint32_t a = smem_addr(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(a, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        record_timeout(site);
        return false;
      }
    }
  }
}

// Short wait used only while draining after an abort.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_addr(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > kDrainLimitNs) return;
  }
}

// ------------------------------------------------------------------ MMA helpers

// S[128 x 128] = Q[128 x D] . K[128 x D]^T; both tiles K-major, 128B-swizzled,
// stored as D/64 panels of 128 rows x 128 bytes. q_lo / k_lo: low descriptor
// words of the tiles (desc_lo_sw128 with LBO 16); a k-step of 16 columns is
// +32 bytes inside a panel, the next panel +kPanelBytes.
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_lo, uint32_t k_lo) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * Cfg<D>::kPanelBytes + (kk & 3) * 32) >> 4;
    mma_ss(d_tmem, desc_join(q_lo + off, kDescHiSw128), desc_join(k_lo + off, kDescHiSw128),
           Cfg<D>::kIdescS, kk > 0 ? 1u : 0u);
  }
}

// O[128 x D] (+)= P[128 x 128] (bf16 in TMEM, 2 per column) . V[128 x D];
// V is MN-major (D contiguous per key row): 16 keys per step = 16 rows = 2048
// bytes. v_lo: low descriptor word of the V tile (LBO = one panel).
template <int D, int K0 = 0, int K1 = BN / 16>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_lo,
                                         uint32_t accumulate) {
#pragma unroll
  for (int kk = K0; kk < K1; ++kk) {
    mma_ts(d_tmem, p_tmem + kk * 8, desc_join(v_lo + kk * (2048 >> 4), kDescHiSw128),
           Cfg<D>::kIdescO, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Bits [0, n) of a 32-bit word, n clamped to [0, 32].
__device__ __forceinline__ uint32_t range_bits(int n) {
  n = n < 0 ? 0 : (n > 32 ? 32 : n);
  return n == 32 ? 0xFFFFFFFFu : ((1u << n) - 1u);
}

__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31]));
}

// ------------------------------------------------------------------ roles

template <int D>
__device__ __forceinline__ void producer_role(const AttnParams& p, Bars<Cfg<D>::kStages>* bars,
                                              uint8_t* smem, const CUtensorMap* tq,
                                              const CUtensorMap* tk, const CUtensorMap* tv) {
  constexpr int NST = Cfg<D>::kStages;
  volatile int* abort_flag = &bars->abort_flag;
  const uint32_t q0 = smem_addr(smem);
  const uint32_t ring = smem_addr(smem + Cfg<D>::kRingOff);
  uint32_t kv_cnt = 0, it_cnt = 0;
  bool ok = true;
  const int n_work = work_count(p, blockIdx.x, gridDim.x);
  // Publishes item k's descriptor (or the end marker) for the softmax warpgroups.
  auto publish = [&](int k, const Item& it, bool end) -> bool {
    const int slot = k % kDescRing;
    if (!wait_bar(&bars->desc_empty[slot], ((k / kDescRing) & 1) ^ 1, abort_flag, kSiteDescEmpty))
      return false;
    ItemDesc& d = bars->desc[slot];
    d.b = it.b; d.g = it.g; d.qb = end ? -1 : it.qb; d.h0 = it.h0; d.h1 = it.h1; d.v1 = it.v1;
    d.t0 = it.t0; d.t1 = it.t1; d.split = it.split; d.hunit = it.hunit;
    mbar_arrive(&bars->desc_full[slot]);  // release: the descriptor is visible to the waiters
    return true;
  };
  // Per item: the first K/V tile goes into the ring before the wait for the Q
  // buffer (its ring slot frees about a tile earlier than the previous item's
  // last S releases Q, so it is in flight before Q), then Q, then the other
  // tiles. The ring order the issuer consumes is unchanged. (An L2 prefetch of
  // the next item's Q on top of this measured within noise and was dropped.)
  auto load_kv = [&](const Item& it, const TileSrc& bt, int t) -> bool {
    const int kb = bt.kb(t);
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const uint32_t st = kv_cnt % NST;
      if (!wait_bar(&bars->kv_empty[st], ((kv_cnt / NST) & 1u) ^ 1u, abort_flag, kSiteKvEmpty))
        return false;
      mbar_arrive_expect_tx(&bars->kv_full[st], Cfg<D>::kTileBytes);
#pragma unroll
      for (int pn = 0; pn < Cfg<D>::kPanels; ++pn)
        tma_load_4d(ring + st * Cfg<D>::kTileBytes + pn * Cfg<D>::kPanelBytes, which ? tv : tk,
                    &bars->kv_full[st], pn * 64, it.g, kb * BN, it.b);
      ++kv_cnt;
    }
    return true;
  };
  for (int k = 0; ok && k < n_work; ++k) {
    const Item it = work_item_at(p, blockIdx.x, gridDim.x, k);
    if (!(ok = publish(k, it, false))) break;
    const TileSrc bt = tile_src(p, it);
    const int t_end = imin(bt.count(), it.t1);
    if (t_end <= it.t0) continue;  // an empty block-sparse list: nothing to load
    if (!(ok = load_kv(it, bt, it.t0))) break;
    if (p.inject_cta == static_cast<int>(blockIdx.x) && it_cnt == 0) {
      ok = false;  // test hook: no Q for the first item (drained and left below)
      break;
    }
    if (!(ok = wait_bar(&bars->q_empty, (it_cnt & 1u) ^ 1u, abort_flag, kSiteQEmpty))) break;
    bars->item_T = t_end - it.t0;
    bars->item_v1 = it.v1;
    mbar_arrive_expect_tx(&bars->q_full, (1 + it.v1) * Cfg<D>::kTileBytes);
#pragma unroll
    for (int pn = 0; pn < Cfg<D>::kPanels; ++pn) {
      tma_load_4d(q0 + pn * Cfg<D>::kPanelBytes, tq, &bars->q_full, pn * 64, it.h0, it.qb * BM, it.b);
      if (it.v1)
        tma_load_4d(q0 + Cfg<D>::kTileBytes + pn * Cfg<D>::kPanelBytes, tq, &bars->q_full, pn * 64,
                    it.h1, (it.qb + p.qpair) * BM, it.b);
    }
    ++it_cnt;
    for (int t = it.t0 + 1; ok && t < t_end; ++t) ok = load_kv(it, bt, t);
  }
  if (ok) ok = publish(n_work, Item{}, true);  // the softmax warpgroups' end marker
  if (ok) {  // no more items: a descriptor of zero tiles, once Q is released
    if ((ok = wait_bar(&bars->q_empty, (it_cnt & 1u) ^ 1u, abort_flag, kSiteQEmpty))) {
      bars->item_T = 0;
      bars->item_v1 = 0;
      mbar_arrive(&bars->q_full);
    }
  }
  if (!ok) {  // let copies already in flight land before the CTA goes away
    const uint32_t first = kv_cnt > (uint32_t)NST ? kv_cnt - NST : 0;
    for (uint32_t idx = first; idx < kv_cnt; ++idx)
      drain_wait(&bars->kv_full[idx % NST], (idx / NST) & 1u);
    if (it_cnt) drain_wait(&bars->q_full, (it_cnt - 1) & 1u);
  }
}

// The tcgen05 issuer: one lane of warp 9 issues every MMA of both Q tiles in the order
// O0+=P0.V_t, S0=Q0.K_{t+1}, O1+=P1.V_t, S1=Q1.K_{t+1}, and keeps that order
// across item boundaries: after the last O0+=P0.V of an item it issues the
// next item's first S0 (then, after O1+=P1.V, its S1), so one softmax
// warpgroup starts the next item while the tensor core finishes the other's
// products. (The next Q is loaded once the current item's last S is done;
// K/V arrive in the ring in exactly this order; the producer publishes each
// item's tile count with its Q, and a zero count after the last item.)
// Descriptors are kept as
// precomputed low words plus per-k-step constant adds: the issuing warp shares
// its SM sub-partition with two softmax warps, so every instruction it saves
// per MMA shortens the time the tensor pipe waits for the next one.
template <int D>
__device__ __forceinline__ void mma_role(const AttnParams& p, Bars<Cfg<D>::kStages>* bars,
                                         uint8_t* smem, uint32_t tmem_base) {
  constexpr int NST = Cfg<D>::kStages;
  // The whole warp runs this loop in step (waits, counters, descriptors), and
  // one lane, elected once, issues every MMA and commit: a commit tracks only
  // the MMAs of the thread that issues it. Keeping the warp converged lets the
  // operands live in uniform registers, so an MMA costs few issue slots on a
  // sub-partition that two softmax warps keep busy.
  const bool leader = elect_one();
  volatile int* abort_flag = &bars->abort_flag;
  const uint32_t q0 = desc_lo_sw128(smem_addr(smem), 16), q1 = desc_lo_sw128(smem_addr(smem) + Cfg<D>::kTileBytes, 16);
  const uint32_t ring = smem_addr(smem + Cfg<D>::kRingOff);
  const uint32_t k_lo0 = desc_lo_sw128(ring, 16);
  const uint32_t v_lo0 = desc_lo_sw128(ring, Cfg<D>::kPanelBytes);
  constexpr uint32_t kStageLo = Cfg<D>::kTileBytes >> 4;
  const uint32_t tS0 = tmem_base + Cfg<D>::kTmemS0, tS1 = tmem_base + Cfg<D>::kTmemS1;
  const uint32_t tO0 = tmem_base + Cfg<D>::kTmemO0, tO1 = tmem_base + Cfg<D>::kTmemO1;
  uint32_t kv_cnt = 0, it_cnt = 0, pc0 = 0, pc1 = 0, oe0 = 0, oe1 = 0;
  bool ok = true;
#define TM_WAIT(bar, par, site)                                                            \
  if (!(ok = __all_sync(0xffffffffu, wait_bar((bar), (par), abort_flag, (site))))) break; \
  tc_fence_after();
  // Items come from the producer's descriptors (no work cursor here: the
  // issuer's registers are few and its loop is on the critical path).
  if (!(ok = __all_sync(0xffffffffu, wait_bar(&bars->q_full, it_cnt & 1u, abort_flag, kSiteQFull)))) {
    if (leader) mma_commit(&bars->mma_done);
    __syncwarp();
    drain_wait(&bars->mma_done, 0);
    return;
  }
  tc_fence_after();
  ++it_cnt;
  int T = bars->item_T;
  bool v1 = bars->item_v1 != 0;
  bool started = false;  // this item's first S products were issued by the previous item's tail
  uint32_t kst = 0;
  while (ok && T > 0) {
    if (!started) {
      kst = kv_cnt % NST;
      TM_WAIT(&bars->kv_full[kst], (kv_cnt / NST) & 1u, kSiteKvFull);
      if (leader) issue_qk<D>(tS0, q0, k_lo0 + kst * kStageLo);
      __syncwarp();
      if (leader) mma_commit(&bars->s_full[0]);
      __syncwarp();
      if (v1) {
        if (leader) issue_qk<D>(tS1, q1, k_lo0 + kst * kStageLo);
        __syncwarp();
        if (leader) mma_commit(&bars->s_full[1]);
        __syncwarp();
      }
      if (T == 1 && leader) mma_commit(&bars->q_empty);
      __syncwarp();
      if (leader) mma_commit(&bars->kv_empty[kst]);
      __syncwarp();
      ++kv_cnt;
    }
    int Tn = 0;
    bool v1n = false;
    // steady state: tiles 0 .. T-2 (the next S of each is this item's tile t+1)
    for (int t = 0; t + 1 < T; ++t) {
      const uint32_t vst = kv_cnt % NST;
      TM_WAIT(&bars->kv_full[vst], (kv_cnt / NST) & 1u, kSiteKvFull);
      if (t == 0) {
        TM_WAIT(&bars->o_empty[0], (oe0 & 1u) ^ 1u, kSiteOEmpty);
        ++oe0;
      }
      TM_WAIT(&bars->p_full[0], pc0 & 1u, kSitePFull);
      if (leader) issue_pv<D, 0, 4>(tO0, tS0, v_lo0 + vst * kStageLo, t > 0 ? 1u : 0u);
      __syncwarp();
      TM_WAIT(&bars->p_full[1], pc0 & 1u, kSitePFull);
      ++pc0;
      if (leader) issue_pv<D, 4, 8>(tO0, tS0, v_lo0 + vst * kStageLo, 1u);
      __syncwarp();
      const uint32_t kidx = kv_cnt + 1;
      kst = kidx % NST;
      TM_WAIT(&bars->kv_full[kst], (kidx / NST) & 1u, kSiteKvFull);
      if (leader) issue_qk<D>(tS0, q0, k_lo0 + kst * kStageLo);
      __syncwarp();
      if (leader) mma_commit(&bars->s_full[0]);
      __syncwarp();
      if (!v1 && t + 1 == T - 1 && leader) mma_commit(&bars->q_empty);
      __syncwarp();
      if (v1) {
        if (t == 0) {
          TM_WAIT(&bars->o_empty[1], (oe1 & 1u) ^ 1u, kSiteOEmpty);
          ++oe1;
        }
        TM_WAIT(&bars->p_full[2], pc1 & 1u, kSitePFull);
        if (leader) issue_pv<D, 0, 4>(tO1, tS1, v_lo0 + vst * kStageLo, t > 0 ? 1u : 0u);
        __syncwarp();
        TM_WAIT(&bars->p_full[3], pc1 & 1u, kSitePFull);
        ++pc1;
        if (leader) issue_pv<D, 4, 8>(tO1, tS1, v_lo0 + vst * kStageLo, 1u);
        __syncwarp();
      }
      if (leader) mma_commit(&bars->kv_empty[vst]);  // V_t free once both P.V products are done
      __syncwarp();
      ++kv_cnt;
      if (v1) {
        if (leader) issue_qk<D>(tS1, q1, k_lo0 + kst * kStageLo);
        __syncwarp();
        if (leader) mma_commit(&bars->s_full[1]);
        __syncwarp();
        if (t + 1 == T - 1 && leader) mma_commit(&bars->q_empty);
        __syncwarp();
      }
      if (leader) mma_commit(&bars->kv_empty[kst]);  // K_{t+1} free once both Q.K products are done
      __syncwarp();
      ++kv_cnt;
    }
    if (!ok) break;
    // last tile: its products, with the next item's first S products in between
    do {
      const int t = T - 1;
      const uint32_t vst = kv_cnt % NST;
      TM_WAIT(&bars->kv_full[vst], (kv_cnt / NST) & 1u, kSiteKvFull);
      if (t == 0) {
        TM_WAIT(&bars->o_empty[0], (oe0 & 1u) ^ 1u, kSiteOEmpty);
        ++oe0;
      }
      TM_WAIT(&bars->p_full[0], pc0 & 1u, kSitePFull);
      if (leader) issue_pv<D, 0, 4>(tO0, tS0, v_lo0 + vst * kStageLo, t > 0 ? 1u : 0u);
      __syncwarp();
      TM_WAIT(&bars->p_full[1], pc0 & 1u, kSitePFull);
      ++pc0;
      if (leader) issue_pv<D, 4, 8>(tO0, tS0, v_lo0 + vst * kStageLo, 1u);
      __syncwarp();
      if (leader) mma_commit(&bars->o_full[0]);
      __syncwarp();
      // the next item's descriptor (and Q), then its S0
      TM_WAIT(&bars->q_full, it_cnt & 1u, kSiteQFull);
      ++it_cnt;
      Tn = bars->item_T;
      v1n = bars->item_v1 != 0;
      if (Tn > 0) {
        const uint32_t kidx = kv_cnt + 1;
        kst = kidx % NST;
        TM_WAIT(&bars->kv_full[kst], (kidx / NST) & 1u, kSiteKvFull);
        if (leader) issue_qk<D>(tS0, q0, k_lo0 + kst * kStageLo);
        __syncwarp();
        if (leader) mma_commit(&bars->s_full[0]);
        __syncwarp();
        if (!v1n && Tn == 1 && leader) mma_commit(&bars->q_empty);
        __syncwarp();
      }
      if (v1) {
        if (t == 0) {
          TM_WAIT(&bars->o_empty[1], (oe1 & 1u) ^ 1u, kSiteOEmpty);
          ++oe1;
        }
        TM_WAIT(&bars->p_full[2], pc1 & 1u, kSitePFull);
        if (leader) issue_pv<D, 0, 4>(tO1, tS1, v_lo0 + vst * kStageLo, t > 0 ? 1u : 0u);
        __syncwarp();
        TM_WAIT(&bars->p_full[3], pc1 & 1u, kSitePFull);
        ++pc1;
        if (leader) issue_pv<D, 4, 8>(tO1, tS1, v_lo0 + vst * kStageLo, 1u);
        __syncwarp();
        if (leader) mma_commit(&bars->o_full[1]);
        __syncwarp();
      }
      if (leader) mma_commit(&bars->kv_empty[vst]);
      __syncwarp();
      ++kv_cnt;
      if (Tn > 0) {
        if (v1n) {
          if (leader) issue_qk<D>(tS1, q1, k_lo0 + kst * kStageLo);
          __syncwarp();
          if (leader) mma_commit(&bars->s_full[1]);
          __syncwarp();
          if (Tn == 1 && leader) mma_commit(&bars->q_empty);
          __syncwarp();
        }
        if (leader) mma_commit(&bars->kv_empty[kst]);
        __syncwarp();
        ++kv_cnt;
      }
    } while (false);
    if (!ok) break;
    T = Tn;
    v1 = v1n;
    started = true;
  }
#undef TM_WAIT
  // Every MMA issued above must finish before TMEM is released.
  if (leader) mma_commit(&bars->mma_done);
  __syncwarp();
  drain_wait(&bars->mma_done, 0);
}

// Split pieces of a heavy item: this warp's 32 rows of the piece's partial
// (unnormalised O, running max m, sum l, all in the log2 domain of m) go to its
// record; record layout: O as float4[D/4][128] (a warp's 16-byte stores cover
// 512 contiguous bytes), then m[128], l[128]. The warp then counts itself in
// its counter; the warp that arrives last (no waiting: the others leave)
// merges all nsplit partials in split order, so the result does not depend on
// which piece finished last, and returns true with orr / l_run replaced by the
// merged O and l. No thread ever waits on another CTA.
template <int D>
__device__ __forceinline__ bool merge_split(const AttnParams& p, const Item& it, int wg, int wq,
                                            int lane, uint32_t (&orr)[D / 32][32], float m_run,
                                            float& l_run) {
  constexpr int kRecFloats = 128 * D + 256;
  const int r = wq * 32 + lane;
  float* recs = p.ws_rec + static_cast<size_t>(it.hunit) * p.nsplit * 2 * kRecFloats;
  {
    float* rec = recs + static_cast<size_t>(it.split * 2 + wg) * kRecFloats;
    float4* ro = reinterpret_cast<float4*>(rec);
#pragma unroll
    for (int c = 0; c < D / 32; ++c)
#pragma unroll
      for (int x = 0; x < 8; ++x)
        __stcg(ro + (c * 8 + x) * 128 + r,
               make_float4(__uint_as_float(orr[c][4 * x]), __uint_as_float(orr[c][4 * x + 1]),
                           __uint_as_float(orr[c][4 * x + 2]), __uint_as_float(orr[c][4 * x + 3])));
    __stcg(rec + 128 * D + r, m_run);
    __stcg(rec + 128 * D + 128 + r, l_run);
  }
  __threadfence();
  __syncwarp();
  int last = 0;
  if (lane == 0) {
    last = atomicAdd(p.ws_cnt + (it.hunit * 2 + wg) * 4 + wq, 1) == p.nsplit - 1;
    __threadfence();
  }
  if (!__shfl_sync(0xffffffffu, last, 0)) return false;
  float M = -INFINITY;
  for (int sp = 0; sp < p.nsplit; ++sp)
    M = fmaxf(M, __ldcg(recs + static_cast<size_t>(sp * 2 + wg) * kRecFloats + 128 * D + r));
  float acc[D / 32][32];
#pragma unroll
  for (int c = 0; c < D / 32; ++c)
#pragma unroll
    for (int x = 0; x < 32; ++x) acc[c][x] = 0.f;
  float l_sum = 0.f;
#pragma unroll 1
  for (int sp = 0; sp < p.nsplit; ++sp) {
    const float* rec = recs + static_cast<size_t>(sp * 2 + wg) * kRecFloats;
    const float ms = __ldcg(rec + 128 * D + r);
    const float w = ms == -INFINITY ? 0.f : ex2(ms - M);
    l_sum = fmaf(w, __ldcg(rec + 128 * D + 128 + r), l_sum);
    const float4* ro = reinterpret_cast<const float4*>(rec);
#pragma unroll
    for (int c = 0; c < D / 32; ++c)
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const float4 v = __ldcg(ro + (c * 8 + x) * 128 + r);
        acc[c][4 * x] = fmaf(w, v.x, acc[c][4 * x]);
        acc[c][4 * x + 1] = fmaf(w, v.y, acc[c][4 * x + 1]);
        acc[c][4 * x + 2] = fmaf(w, v.z, acc[c][4 * x + 2]);
        acc[c][4 * x + 3] = fmaf(w, v.w, acc[c][4 * x + 3]);
      }
  }
#pragma unroll
  for (int c = 0; c < D / 32; ++c)
#pragma unroll
    for (int x = 0; x < 32; ++x) orr[c][x] = __float_as_uint(acc[c][x]);
  l_run = l_sum;
  return true;
}

template <int D>
__device__ __forceinline__ void softmax_role(const AttnParams& p, Bars<Cfg<D>::kStages>* bars,
                                             uint8_t* smem, const CUtensorMap* to, int wg, int wq,
                                             int lane, uint32_t tmem_base) {
  volatile int* abort_flag = &bars->abort_flag;
  const int r = wq * 32 + lane;  // row of the Q tile == TMEM lane
  const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
  const uint32_t tS = tmem_base + lane_addr + (wg ? Cfg<D>::kTmemS1 : Cfg<D>::kTmemS0);
  const uint32_t tO = tmem_base + lane_addr + (wg ? Cfg<D>::kTmemO1 : Cfg<D>::kTmemO0);
  const float sl2 = p.sl2;
  uint32_t s_cnt = 0, o_cnt = 0;
  for (int k = 0;; ++k) {
    // the producer's descriptor of this CTA's next item (qb < 0: no more)
    const int ds = k % kDescRing;
    const bool okd = wait_bar(&bars->desc_full[ds], (k / kDescRing) & 1, abort_flag, kSiteDescFull);
    if (!__all_sync(0xffffffffu, okd)) return;
    Item it;
    {
      const ItemDesc& d = bars->desc[ds];
      it.b = d.b; it.g = d.g; it.qb = d.qb; it.h0 = d.h0; it.h1 = d.h1; it.v1 = d.v1;
      it.t0 = d.t0; it.t1 = d.t1; it.split = d.split; it.hunit = d.hunit;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->desc_empty[ds]);
    if (it.qb < 0) break;
    if (wg == 1 && !it.v1) continue;
    const TileSrc bt = tile_src(p, it);
    const int T = imin(bt.count(), it.t1) - it.t0;
    const int head = wg ? it.h1 : it.h0;
    const Pattern pat = head_pattern(p, head);  // this Q tile's own mask
    const int my_qb = it.qb + (p.qpair ? wg : 0);  // this Q tile's q-block
    const int i = my_qb * BM + r;  // query row of this thread
    // kept keys of row i: [0, sink_hi) U [band_lo, hi)
    const int hi = imin(i, pat.N - 1) + 1;
    const bool full_row = pat.causal || i >= pat.N - pat.L;
    const int sink_hi = full_row ? hi : imin(pat.S, hi);
    const int band_lo = full_row ? hi : imax(0, i - pat.W + 1);
    float m_run = -INFINITY, l_run = 0.f;
    for (int t = 0; t < T; ++t) {
      const int kb = bt.kb(it.t0 + t);  // read before the wait, which hides its latency
      const bool bad = kb < 0;          // a clamped negative index entry: fully masked
      const bool need_mask = bad || tile_needs_mask(pat, my_qb, kb, BM, BN) != 0;
      bool ok = wait_bar(&bars->s_full[wg], s_cnt & 1u, abort_flag, kSiteSFull);
      ++s_cnt;
      if (!__all_sync(0xffffffffu, ok)) return;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, sr[c]);
      tmem_wait_ld(sr[0]);
      reg_fence(sr[1]);
      reg_fence(sr[2]);
      reg_fence(sr[3]);
      if (need_mask) {
        // keep bits of this row for the tile's 128 columns, then -inf elsewhere
        const int c0 = bad ? (1 << 30) : kb * BN;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t keep = range_bits(sink_hi - c0 - 32 * c) |
                                (range_bits(hi - c0 - 32 * c) & ~range_bits(band_lo - c0 - 32 * c));
#pragma unroll
          for (int x = 0; x < 32; ++x)
            sr[c][x] = ((keep >> x) & 1u) ? sr[c][x] : 0xFF800000u;
        }
      }
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int x = 0; x < 32; ++x) s[32 * c + x] = __uint_as_float(sr[c][x]);
      // row max: 3-input max over eight independent chains
      float mxa[8];
#pragma unroll
      for (int y = 0; y < 8; ++y) mxa[y] = fmaxf(s[2 * y], s[2 * y + 1]);
#pragma unroll
      for (int x = 16; x < 128; x += 16)
#pragma unroll
        for (int y = 0; y < 8; ++y) mxa[y] = fmax3(mxa[y], s[x + 2 * y], s[x + 2 * y + 1]);
      const float mx = fmaxf(fmax3(mxa[0], mxa[1], mxa[2]),
                             fmax3(fmax3(mxa[3], mxa[4], mxa[5]), mxa[6], mxa[7]));
      const float m_new = fmaxf(m_run, mx * sl2);
      const bool bump = m_new > m_run + kRescaleThreshold;
      float alpha = 1.f;
      if (bump) {
        alpha = ex2(m_run - (m_new + kRescaleMargin));
        m_run = m_new + kRescaleMargin;
      }
      const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
      // O must be rescaled before the first half of this tile's P.V is issued
      if (t > 0 && __any_sync(0xffffffffu, bump)) {
#pragma unroll 1
        for (int c = 0; c < D / 16; ++c) {  // 16 columns at a time: the scores are still live
          uint32_t orr[16];
          tmem_ld16(tO + 16 * c, orr);
          tmem_wait_ld16(orr);
#pragma unroll
          for (int x = 0; x < 16; ++x) orr[x] = __float_as_uint(__uint_as_float(orr[x]) * alpha);
          tmem_st16(tO + 16 * c, orr);
        }
      }
      // p = 2^(s * scale * log2 e - m): packed fp32x2 FMA, then exp2; l sums the
      // same bf16-rounded weights that P.V uses (exact widening adds), so O / l is
      // a properly normalised average of v (a single dominant key returns v exactly;
      // summing the unrounded fp32 weights instead saves an instruction per pair
      // but leaves O off by up to 2^-9 of |v| for peaked rows, which outlier-channel
      // inputs push past the tolerance once the bf16 output rounding is added).
      // P is published in two halves (keys 0-63, 64-127): the MMA issuer starts
      // the first half of P.V while the second half is still being exponentiated.
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          // the first kPolyPairs pairs of every 32 use the FMA-pipe exp2, the rest MUFU
          float xa, xb;
          ffma2(xa, xb, s[64 * h + 2 * x], s[64 * h + 2 * x + 1], sl2, sl2, neg_m, neg_m);
          float a, b;
          if (x < kPolyPairs) {
            ex2x2_poly(a, b, xa, xb);
          } else {
            a = ex2(xa);
            b = ex2(xb);
          }
          pk[x] = pack_bf16x2(a, b);
          add_bf16x2_to_f32(acc[2 * (x & 3)], acc[2 * (x & 3) + 1], pk[x]);
        }
        tmem_st32(tS + 32 * h, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[2 * wg + h]);
      }
      const float rs = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
      l_run = l_run * alpha + rs;
    }
    // epilogue: O / l -> bf16 -> this warp's 128B-swizzled staging slot (32 rows x
    // 64 columns at a time) -> one TMA store per half; rows past N are clipped.
    uint32_t orr[D / 32][32];
    if (T > 0) {
      bool ok = wait_bar(&bars->o_full[wg], o_cnt & 1u, abort_flag, kSiteOFull);
      ++o_cnt;
      if (!__all_sync(0xffffffffu, ok)) return;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + 32 * c, orr[c]);
      tmem_wait_ld(orr[0]);
#pragma unroll
      for (int c = 1; c < D / 32; ++c) reg_fence(orr[c]);
      tc_fence_before();
      mbar_arrive(&bars->o_empty[wg]);
    } else {  // an empty block-sparse list: the rows keep no key and come out as zeros
#pragma unroll
      for (int c = 0; c < D / 32; ++c)
#pragma unroll
        for (int x = 0; x < 32; ++x) orr[c][x] = 0u;
    }
    if (it.split >= 0 && !merge_split<D>(p, it, wg, wq, lane, orr, m_run, l_run)) continue;
    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
    const uint32_t slot = smem_addr(smem + Cfg<D>::kStageOff) + (wg * 4 + wq) * Cfg<D>::kStageSlotBytes;
    const uint32_t row_addr = slot + lane * 128;
#pragma unroll
    for (int h = 0; h < D / 64; ++h) {
      if (lane == 0) bulk_wait_read_all();  // the slot's previous store has read it
      __syncwarp();
#pragma unroll
      for (int x = 0; x < 8; ++x) {  // 16-byte chunk x holds columns 64h + 8x .. 64h + 8x + 7
        const int c = 2 * h + (x >> 2), o = (8 * x) & 31;
        st_shared_v4(row_addr + ((x ^ (lane & 7)) << 4),
                     pack_bf16x2(__uint_as_float(orr[c][o]) * inv_l, __uint_as_float(orr[c][o + 1]) * inv_l),
                     pack_bf16x2(__uint_as_float(orr[c][o + 2]) * inv_l, __uint_as_float(orr[c][o + 3]) * inv_l),
                     pack_bf16x2(__uint_as_float(orr[c][o + 4]) * inv_l, __uint_as_float(orr[c][o + 5]) * inv_l),
                     pack_bf16x2(__uint_as_float(orr[c][o + 6]) * inv_l, __uint_as_float(orr[c][o + 7]) * inv_l));
      }
      fence_proxy_async_smem();  // make the generic-proxy writes visible to the TMA engine
      __syncwarp();
      if (lane == 0 && my_qb * BM + wq * 32 < p.N) {  // a slot wholly past N stores nothing
        tma_store_4d(to, slot, 64 * h, head, my_qb * BM + wq * 32, it.b);
        bulk_commit_group();
      }
    }
  }
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_addr(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                const __grid_constant__ AttnParams p) {
  constexpr int NST = Cfg<D>::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  auto* bars = reinterpret_cast<Bars<NST>*>(smem + Cfg<D>::kBarOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars->s_full[w], 1);
      mbar_init(&bars->p_full[2 * w], 128);
      mbar_init(&bars->p_full[2 * w + 1], 128);
      mbar_init(&bars->o_full[w], 1);
      mbar_init(&bars->o_empty[w], 128);
    }
    mbar_init(&bars->mma_done, 1);
    for (int r = 0; r < kDescRing; ++r) {
      mbar_init(&bars->desc_full[r], 1);
      mbar_init(&bars->desc_empty[r], 8);  // one arrival per softmax warp
    }
    bars->abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpTma && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    tma_prefetch_desc(&to);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  if (warp < 8) {
    setmaxnreg_inc<kSoftmaxRegs>();
    softmax_role<D>(p, bars, smem, &to, warp >> 2, warp & 3, lane, tmem_base);
    if (lane == 0) bulk_wait_all();  // output stores done before shared memory goes away
    __syncwarp();
  } else {
    setmaxnreg_dec<kSideRegs>();
  }
  if (warp < 8) {
  } else if (warp == kWarpTma) {
    if (lane == 0) producer_role<D>(p, bars, smem, &tq, &tk, &tv);
    __syncwarp();
  } else if (warp == kWarpMma) {
    mma_role<D>(p, bars, smem, tmem_base);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------ debug kernels

__global__ void dump_tiles_kernel(Pattern pat, int nqb, int* out, long long cap) {
  const int qb = blockIdx.x * blockDim.x + threadIdx.x;
  if (qb >= nqb) return;
  long long off = 0;
  for (int q = 0; q < qb; ++q) off += block_tiles(pat, q, BM, BN).count();
  const BlockTiles bt = block_tiles(pat, qb, BM, BN);
  for (int t = 0; t < bt.count(); ++t) {
    const long long rec = off + t;
    if (rec >= cap) return;
    const int kb = bt.kb(t);
    out[3 * rec + 0] = qb;
    out[3 * rec + 1] = kb;
    out[3 * rec + 2] = tile_full(pat, qb, kb, BM, BN);
  }
}

template <int D>
__global__ void __launch_bounds__(128, 1)
    mma_probe_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, float* s_out, float* o_out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  constexpr int TB = Cfg<D>::kTileBytes;
  uint64_t* bar_load = reinterpret_cast<uint64_t*>(smem + 3 * TB);
  uint64_t* bar_mma = bar_load + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_load + 2);
  int* abort_flag = reinterpret_cast<int*>(bar_load + 3);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t sq = smem_addr(smem), sk = sq + TB, sv = sq + 2 * TB;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar_load, 3 * TB);
    for (int pn = 0; pn < Cfg<D>::kPanels; ++pn) {
      tma_load_4d(sq + pn * Cfg<D>::kPanelBytes, &tq, bar_load, pn * 64, 0, 0, 0);
      tma_load_4d(sk + pn * Cfg<D>::kPanelBytes, &tk, bar_load, pn * 64, 0, 0, 0);
      tma_load_4d(sv + pn * Cfg<D>::kPanelBytes, &tv, bar_load, pn * 64, 0, 0, 0);
    }
  }
  bool ok = wait_bar(bar_load, 0, abort_flag, kSiteProbe);
  if (threadIdx.x == 0 && ok) {
    tc_fence_after();
    issue_qk<D>(tbase, desc_lo_sw128(sq, 16), desc_lo_sw128(sk, 16));
    mma_commit(bar_mma);
  }
  ok = ok && wait_bar(bar_mma, 0, abort_flag, kSiteProbe);
  ok = __all_sync(0xffffffffu, ok);
  const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
  const int r = threadIdx.x;
  if (ok) {
    tc_fence_after();
    uint32_t sr[4][32];
    for (int c = 0; c < 4; ++c) tmem_ld32(tbase + lane_addr + 32 * c, sr[c]);
    tmem_wait_ld(sr[0]);
    reg_fence(sr[1]);
    reg_fence(sr[2]);
    reg_fence(sr[3]);
    for (int c = 0; c < 4; ++c)
      for (int x = 0; x < 32; ++x) s_out[r * 128 + 32 * c + x] = __uint_as_float(sr[c][x]);
    for (int h = 0; h < 2; ++h) {
      uint32_t pk[32];
      for (int x = 0; x < 32; ++x)
        pk[x] = pack_bf16x2(__uint_as_float(sr[2 * h + (x >> 4)][(2 * x) & 31]),
                            __uint_as_float(sr[2 * h + (x >> 4)][(2 * x + 1) & 31]));
      tmem_st32(tbase + lane_addr + 32 * h, pk);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && ok) {
    tc_fence_after();
    issue_pv<D>(tbase + 128, tbase, desc_lo_sw128(sv, Cfg<D>::kPanelBytes), 0u);
    mma_commit(bar_mma);
  }
  ok = ok && wait_bar(bar_mma, 1, abort_flag, kSiteProbe);
  ok = __all_sync(0xffffffffu, ok);
  if (ok) {
    tc_fence_after();
    for (int c = 0; c < D / 32; ++c) {
      uint32_t orr[32];
      tmem_ld32(tbase + lane_addr + 128 + 32 * c, orr);
      tmem_wait_ld(orr);
      for (int x = 0; x < 32; ++x) o_out[r * D + 32 * c + x] = __uint_as_float(orr[x]);
    }
  }
  if (threadIdx.x == 0) {  // nothing may still be in flight when TMEM is freed
    mma_commit(bar_mma);
    drain_wait(bar_mma, ok ? 0u : 1u);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

// ------------------------------------------------------------------ pattern discovery

#include "tm_discover.cuh"

// ------------------------------------------------------------------ host side

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Per-device facts. ready / supported / sms are written once under g_mutex and
// read by callers that went through device_info (which takes it); the
// per-kernel "shared-memory attribute set" flags are atomics, set under
// g_mutex after the attribute call and read without it.
struct DeviceInfo {
  bool ready = false;
  bool supported = false;
  int sms = 0;
  std::atomic<bool> attr_set[2] = {false, false};
  std::atomic<bool> probe_attr_set[2] = {false, false};
  std::atomic<bool> disc_attr_set[2] = {false, false};
};

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
// Kernels this library has launched in the process (every launch site counts
// itself once its launch returned without an error).
std::atomic<long long> g_launches{0};

int counted(int n) {
  if (cudaGetLastError() != cudaSuccess) return TM_ERR_CUDA;
  g_launches.fetch_add(n, std::memory_order_relaxed);
  return TM_OK;
}
EncodeTiledFn g_encode = nullptr;
DeviceInfo g_devices[kMaxDevices];  // fixed: pointers handed out stay valid

// Sets a kernel's dynamic shared-memory limit once per device.
template <class K>
int set_smem_once(std::atomic<bool>& flag, K kernel, int bytes) {
  if (flag.load(std::memory_order_acquire)) return TM_OK;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (flag.load(std::memory_order_relaxed)) return TM_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return TM_ERR_CUDA;
  flag.store(true, std::memory_order_release);
  return TM_OK;
}

int get_encode_fn() {
  if (g_encode) return TM_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return TM_ERR_CUDA;
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  return TM_OK;
}

// Device facts, cached per device (thread-safe).
int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (int rc = get_encode_fn()) return rc;
  DeviceInfo& di = g_devices[dev];
  if (!di.ready) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return TM_ERR_CUDA;
    di.supported = (prop.major == 10 && prop.minor == 0);
    di.sms = prop.multiProcessorCount;
    di.ready = true;
  }
  *out = &di;
  return di.supported ? TM_OK : TM_ERR_UNSUPPORTED;
}

// [B, N, H, D] bf16 tensor, 64-column x 128-row boxes, 128-byte swizzle.
int encode_bnhd(CUtensorMap* m, const void* base, int B, int N, int H, int D, int box_rows) {
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2,
                                 (cuuint64_t)N * H * D * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TM_OK : TM_ERR_CUDA;
}

// Fills the geometry and the persistent work split of *p; returns the grid
// size. split: heavy items may be cut into pieces (the caller has workspace).
// The work is the q-blocks [qb0, qb0 + nqb_w) (nqb_w < 0: to the end).
int build_schedule(int B, int Hq, int Hkv, int N, const Pattern& pat, int max_ctas, bool split,
                   AttnParams* p, bool sparse = false, bool mix_pairs = false, int qb0 = 0,
                   int nqb_w = -1, const int* hS = nullptr, const int* hW = nullptr) {
  p->B = B; p->Hq = Hq; p->Hkv = Hkv; p->N = N;
  p->G = Hq / Hkv;
  p->npairs = (p->G + 1) / 2;
  p->nqb_all = (N + BM - 1) / BM;
  p->qb0 = qb0;
  p->nqb = nqb_w < 0 ? p->nqb_all - qb0 : nqb_w;
  p->units = B * Hkv * p->npairs;
  p->pat = pat;
  p->ws_rec = nullptr;
  p->ws_cnt = nullptr;
  p->pair_rot = 0;
  p->kv_rot = 0;
  p->inject_cta = -1;
  p->bs_off = nullptr;
  p->bs_idx = nullptr;
  p->bs_nnz = 0;
  p->ph = 0;
  p->gchunk = 0;
  p->qchunk = 1;
  p->qpair = 0;
  p->qdelta = 0;
  const bool whole = qb0 == 0 && (nqb_w < 0 || nqb_w == p->nqb_all);
  if (!sparse && whole && ((mix_pairs && !pat.causal) || (pat.causal && !mix_pairs && p->G % 2 == 1 && p->G > 1))) {
    // per-head band launches, and causal launches of odd groups: items are
    // q-block pairs of one head; the first q-block whose list is full causal
    // (it holds last-L rows; q-block 0 in a causal launch) starts a pair
    p->qpair = 1;
    const int kf = (!pat.causal && p->pat.L > 0) ? (N - p->pat.L) / BM : p->nqb_all;
    p->qdelta = kf % 2;
    p->npairs = p->G;
    p->units = B * Hkv * p->npairs;
    p->nqb = (p->nqb_all + p->qdelta + 1) / 2;
  }
  // Persistent grid. Item cost = (visited tiles + fixed per-item overhead,
  // about the pipeline fill/drain and epilogue) x Q tiles of the item; it is
  // used to find the heavy q-blocks, how finely to cut them, and how many
  // rounds the CTAs holding an extra heavy piece sit out.
  const long long n_items = static_cast<long long>(p->nqb) * p->units;
  int grid = static_cast<int>(std::min<long long>(std::min(max_ctas, kMaxCtas), n_items));
  std::vector<long long> qcost(p->nqb);
  long long total = 0;
  // (per-head bands: the heavy items and the split are chosen from the costs
  // at the maximal band, as the workspace query sees them; the rounds the
  // CTAs holding an extra heavy item sit out are counted from the heads' own
  // mean costs, in mcost)
  // (with q-block pairs an item holds 1 or 2 Q tiles, one item per head and
  // pair: the costs below are then per item, both Q tiles included)
  std::vector<long long> mcost(p->nqb);
  for (int qb = 0; qb < p->nqb; ++qb) {
    const int x = p->qb0 + qb, qa = 2 * x - p->qdelta;
    const int nq = p->qpair ? (qa >= 0 ? 1 : 0) + (qa + 1 < p->nqb_all ? 1 : 0) : 1;
    qcost[qb] = (sched_tiles(*p, p->pat, x).count() + kItemOverheadTiles) * nq;
    total += qcost[qb] * static_cast<long long>(B) * Hq;
    mcost[qb] = qcost[qb];
    if (hS && hW) {
      long long sum = 0;
      for (int h = 0; h < Hq; ++h)
        sum += sched_tiles(*p, make_pattern(N, 0, hS[h], hW[h], pat.L), x).count();
      mcost[qb] = ((sum + Hq / 2) / Hq + kItemOverheadTiles) * nq;
    }
  }
  const double target = static_cast<double>(total) / grid;
  // heavy q-blocks: from the top, while an item of the block costs more than a
  // quarter of a CTA's share, or more than twice the median q-block (a
  // CTA that drew such an item in the strided rounds would carry its excess;
  // dealt first, its holders join the rounds late instead); at most 8 big
  // items per CTA
  const long long item_q = p->qpair ? 1 : (p->G >= 2 ? 2 : 1);
  std::vector<long long> sorted_cost(qcost);
  std::nth_element(sorted_cost.begin(), sorted_cost.begin() + p->nqb / 2, sorted_cost.end());
  const long long median = sorted_cost[p->nqb / 2];
  // (block-sparse launches: costs are in device memory, every item is dealt
  // in the strided rounds, q-blocks from the last)
  int n_hqb = 0;
  while (!sparse && n_hqb < p->nqb - 1 &&
         (4.0 * qcost[p->nqb - 1 - n_hqb] * item_q > target ||
          qcost[p->nqb - 1 - n_hqb] > 2 * median) &&
         static_cast<long long>(n_hqb + 1) * p->units <= 8LL * grid)
    ++n_hqb;
  p->n_hqb = n_hqb;
  p->n_hunits = n_hqb * p->units;
  // Cut the heavy q-blocks whose items cost more than kSplitShare of a CTA's
  // share into ns pieces (ns from the heaviest, so its pieces fit that share),
  // each of at least kMinPieceTiles tiles, at most 8 big pieces per CTA.
  int ns = 1, n_sqb = 0;
  if (split && !sparse && n_hqb > 0) {
    const double heavy = static_cast<double>(qcost[p->nqb - 1] * item_q);
    ns = static_cast<int>(std::ceil(heavy / (kSplitShare * target)));
    ns = std::min(ns, std::max(1, sched_tiles(*p, p->pat, p->qb0 + p->nqb - 1).count() /
                                      kMinPieceTiles));
    ns = std::min(ns, kMaxSplit);
    while (n_sqb < n_hqb && qcost[p->nqb - 1 - n_sqb] * item_q > kSplitShare * target &&
           sched_tiles(*p, p->pat, p->qb0 + p->nqb - 1 - n_sqb).count() >= ns * kMinPieceTiles)
      ++n_sqb;
    ns = std::min(ns, std::max(1, static_cast<int>(
                              (8LL * grid - (n_hqb - n_sqb) * static_cast<long long>(p->units)) /
                              std::max(1LL, static_cast<long long>(n_sqb) * p->units))));
    if (ns <= 1 || n_sqb == 0) { ns = 1; n_sqb = 0; }
  }
  p->nsplit = ns;
  p->n_sqb = n_sqb;
  p->n_sbig = n_sqb * p->units * ns;
  p->n_big = p->n_sbig + (n_hqb - n_sqb) * p->units;
  // per stride of grid items a digit of radix n advances by d (plus carries)
  // and the q-block slot by d_qi; the first rotation r that makes d + d_qi * r
  // coprime with n lets that digit run through all its values
  // (a stride's q-block slot advance is d_qi, or d_qi + 1 when the lower
  // digits carry; a rotation that makes either advance coprime with n moves
  // the digit through all its values over the CTA's items)
  auto coprime_rotation = [](int d, int d_qi, int n) {
    auto coprime = [](int a, int b) {
      while (b) { const int t = a % b; a = b; b = t; }
      return a == 1;
    };
    for (int r = 0; r < n; ++r)
      if (coprime((d + d_qi * r) % n, n)) return r;
    for (int r = 0; r < n; ++r)
      if (coprime((d + (d_qi + 1) * r) % n, n)) return r;
    return 0;
  };
  // (chunked order: items of one turn must cost alike, so the group is even
  // or its items are q-block pairs)
  if (p->pat.causal && !sparse && !mix_pairs && (p->G % 2 == 0 || p->qpair) && n_hqb == 0 &&
      grid >= p->npairs) {
    p->gchunk = 1;
    p->qchunk = grid / p->npairs;
    // one turn per round exactly: with 7 heads a group's turn is 147 items, and
    // a 148th CTA would shift the turn boundary by one item every round
    grid = p->qchunk * p->npairs;
  }
  const int d_qi = grid / p->units;
  if (!p->gchunk && (p->G % 2 == 1 || mix_pairs) && p->npairs > 1)
    p->pair_rot = coprime_rotation((grid % p->units) % p->npairs, d_qi, p->npairs);
  if (mix_pairs && p->Hkv > 1)
    p->kv_rot = coprime_rotation((grid % p->units) / p->npairs % p->Hkv, d_qi, p->Hkv);
  p->n_a = 0;
  p->n_skip = 0;
  const long long n_norm = n_items - p->n_hunits;
  if (p->n_big % grid != 0 && n_norm > 0) {
    // CTAs [0, n_a) hold one big piece more; they sit out the rounds that the
    // others spend on an equal cost of normal items
    double big_cost = 0, norm_cost = 0;
    for (int q = 0; q < n_hqb; ++q)
      big_cost += mcost[p->nqb - 1 - q] +
                  (q < n_sqb ? ns * kSplitOverheadTiles + (ns - 1) * kItemOverheadTiles : 0);
    big_cost = big_cost * B * Hq / p->n_big;
    for (int qb = 0; qb < p->nqb - n_hqb; ++qb) norm_cost += mcost[qb];
    norm_cost = norm_cost * B * Hq / n_norm;
    p->n_a = p->n_big % grid;
    const double rounds = big_cost / norm_cost;
    const long long max_rounds = n_norm / std::max(1, grid - p->n_a);
    p->n_skip = static_cast<int>(std::min<long long>(max_rounds, static_cast<long long>(rounds + 0.5)));
  }
  return grid;
}

// Workspace of a split schedule: the arrival counters (one int per cut item,
// Q tile and warp, padded to 256 bytes), then one partial record per cut
// item, piece and Q tile. 0 when nothing is split.
struct WsLayout {
  long long cnt_bytes, total;
};
WsLayout ws_layout(const AttnParams& p, int D) {
  WsLayout w{0, 0};
  if (p.nsplit <= 1) return w;
  const long long n_cut = static_cast<long long>(p.n_sqb) * p.units;  // items that are cut
  w.cnt_bytes = (n_cut * 8 * 4 + 255) / 256 * 256;
  const long long rec_bytes = (128LL * D + 256) * 4;
  w.total = w.cnt_bytes + n_cut * p.nsplit * 2 * rec_bytes;
  return w;
}

template <int D>
int launch_attention_d(const LaunchArgs& a, DeviceInfo* di) {
  const int kidx = D == 128 ? 1 : 0;
  if (!di->attr_set[kidx].load(std::memory_order_acquire)) {
    // setmaxnreg redistributes exactly kThreads x kLaunchRegs registers; any
    // other launch register count could leave the increase waiting forever.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, attn_kernel<D>) != cudaSuccess) return TM_ERR_CUDA;
    if (fa.numRegs != kLaunchRegs) {
      fprintf(stderr, "tm: attention kernel built with %d registers, expected %d\n", fa.numRegs,
              kLaunchRegs);
      return TM_ERR_UNSUPPORTED;
    }
    if (int rc = set_smem_once(di->attr_set[kidx], attn_kernel<D>, Cfg<D>::kSmemBytes)) return rc;
  }
  CUtensorMap tq, tk, tv, to;
  if (encode_bnhd(&tq, a.q, a.B, a.N, a.Hq, D, BM) || encode_bnhd(&tk, a.k, a.B, a.N, a.Hkv, D, BN) ||
      encode_bnhd(&tv, a.v, a.B, a.N, a.Hkv, D, BN) || encode_bnhd(&to, a.o, a.B, a.N, a.Hq, D, 32))
    return TM_ERR_CUDA;

  AttnParams p;
  const bool sparse = a.bs_off != nullptr;
  // per-head bands: pairs differ in cost, so every CTA cycles through the pairs
  const int grid = build_schedule(a.B, a.Hq, a.Hkv, a.N, a.pat, di->sms, a.ws != nullptr, &p,
                                  sparse, a.hS != nullptr, a.qb_lo, a.qb_hi - a.qb_lo, a.hS, a.hW);
  p.sl2 = a.scale * 1.4426950408889634f;
  p.inject_cta = a.inject_cta;
  if (a.hS) {  // per-head bands; a.pat already holds the maxima
    if (a.Hq > kMaxBandHeads) return TM_ERR_UNSUPPORTED;
    p.ph = 1;
    for (int h = 0; h < a.Hq; ++h) {
      p.hS[h] = std::min(std::max(a.hS[h], 0), a.N);
      p.hW[h] = std::min(std::max(a.hW[h], 1), a.N);
    }
    const int G = a.Hq / a.Hkv;
    std::vector<int> order(G);
    for (int g = 0; g < a.Hkv; ++g) {  // pair the heads of a group in band order
      for (int x = 0; x < G; ++x) order[x] = g * G + x;
      std::stable_sort(order.begin(), order.end(), [&](int u, int v) {
        return p.hW[u] != p.hW[v] ? p.hW[u] < p.hW[v] : p.hS[u] < p.hS[v];
      });
      for (int x = 0; x < G; ++x) p.hperm[g * G + x] = static_cast<unsigned char>(order[x]);
    }
  }
  if (sparse) {
    p.bs_off = a.bs_off;
    p.bs_idx = a.bs_idx;
    p.bs_nnz = static_cast<int>(a.bs_nnz);
  }
  const WsLayout w = ws_layout(p, D);
  if (w.total > 0) {
    if (a.ws_bytes < w.total) return TM_ERR_INVALID_ARG;
    p.ws_cnt = static_cast<int*>(a.ws);
    p.ws_rec = reinterpret_cast<float*>(static_cast<uint8_t*>(a.ws) + w.cnt_bytes);
    if (cudaMemsetAsync(a.ws, 0, w.cnt_bytes, static_cast<cudaStream_t>(a.stream)) != cudaSuccess)
      return TM_ERR_CUDA;
  }
  attn_kernel<D><<<grid, kThreads, Cfg<D>::kSmemBytes, static_cast<cudaStream_t>(a.stream)>>>(
      tq, tk, tv, to, p);
  return counted(1);
}

// [planes, rows, D] bf16 (D contiguous), 64-column x 128-row boxes, 128-byte swizzle.
int encode_3d(CUtensorMap* m, const void* base, int D, long long rows, long long planes) {
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)planes};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TM_OK : TM_ERR_CUDA;
}

// Discovery workspace: pooled keys, probe rows, scores, counts (256-byte aligned).
struct DiscLayout {
  long long kbar, probes, scores, counts, total;
};
DiscLayout disc_layout(int B, int Hkv, int N, int D, int R) {
  auto al = [](long long x) { return (x + 255) / 256 * 256; };
  const long long lists = static_cast<long long>(B) * Hkv * ((N + BM - 1) / BM);
  const long long nqb = (N + BM - 1) / BM;
  DiscLayout l;
  l.kbar = 0;
  l.probes = l.kbar + al(lists * D * 2);
  l.scores = l.probes + al(lists * R * D * 2);
  l.counts = l.scores + al(lists * nqb * 4);
  l.total = l.counts + al(lists * 4);
  return l;
}

template <int D>
int launch_discovery_d(const DiscArgs& a, DeviceInfo* di) {
  const int kidx = D == 128 ? 1 : 0;
  if (int rc = set_smem_once(di->disc_attr_set[kidx], score_kernel<D>, DiscCfg<D>::kSmem))
    return rc;
  const int G = a.Hq / a.Hkv, R = G * a.P, nqb = (a.N + BM - 1) / BM;
  const DiscLayout l = disc_layout(a.B, a.Hkv, a.N, D, R);
  if (a.ws_bytes < l.total) return TM_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  DiscParams p;
  p.B = a.B; p.Hkv = a.Hkv; p.N = a.N; p.G = G; p.nqb = nqb; p.P = a.P; p.R = R;
  p.qbt = 128 / R;
  p.sl2 = a.scale * 1.4426950408889634f;
  p.alpha = a.alpha;
  p.q = static_cast<const uint16_t*>(a.q);
  p.k = static_cast<const uint16_t*>(a.k);
  p.kbar = reinterpret_cast<uint16_t*>(ws + l.kbar);
  p.probes = reinterpret_cast<uint16_t*>(ws + l.probes);
  p.scores = a.scores_out ? a.scores_out : reinterpret_cast<float*>(ws + l.scores);
  p.counts = reinterpret_cast<int*>(ws + l.counts);
  p.offsets = a.offsets;
  p.indices = a.indices;
  const long long BH = static_cast<long long>(a.B) * a.Hkv;
  CUtensorMap tp, tkb;
  if (encode_3d(&tp, p.probes, D, static_cast<long long>(nqb) * R, BH) ||
      encode_3d(&tkb, p.kbar, D, nqb, BH))
    return TM_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(a.stream);
  const dim3 g1(nqb, static_cast<unsigned>(BH));
  pool_probe_kernel<D><<<g1, kDiscThreads, 0, st>>>(p);
  const dim3 g2((nqb + p.qbt - 1) / p.qbt, static_cast<unsigned>(BH));
  score_kernel<D><<<g2, kDiscThreads, DiscCfg<D>::kSmem, st>>>(tp, tkb, p);
  const long long lists = BH * nqb;
  const unsigned wblocks = static_cast<unsigned>((lists * 32 + 255) / 256);
  count_kernel<<<wblocks, 256, 0, st>>>(p);
  scan_kernel<<<1, 1024, 0, st>>>(p);
  write_index_kernel<<<wblocks, 256, 0, st>>>(p);
  return counted(5);
}

}  // namespace

long long kernel_launches() { return g_launches.load(std::memory_order_relaxed); }

long long discovery_workspace_bytes(int B, int Hq, int Hkv, int N, int D, int P) {
  return disc_layout(B, Hkv, N, D, (Hq / Hkv) * P).total;
}

int launch_discovery(const DiscArgs& a) {
  DeviceInfo* di = nullptr;
  if (int rc = device_info(&di)) return rc;
  if (a.D == 128) return launch_discovery_d<128>(a, di);
  if (a.D == 64) return launch_discovery_d<64>(a, di);
  return TM_ERR_UNSUPPORTED;
}

int launch_attention(const LaunchArgs& a) {
  DeviceInfo* di = nullptr;
  if (int rc = device_info(&di)) return rc;
  if (a.D == 128) return launch_attention_d<128>(a, di);
  if (a.D == 64) return launch_attention_d<64>(a, di);
  return TM_ERR_UNSUPPORTED;
}

int workspace_bytes(int B, int Hq, int Hkv, int N, int D, const Pattern& pat, int num_ctas,
                    long long* bytes) {
  if (num_ctas <= 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&num_ctas, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return TM_ERR_CUDA;
  }
  AttnParams p;
  build_schedule(B, Hq, Hkv, N, pat, num_ctas, true, &p);
  *bytes = ws_layout(p, D).total;
  if (!pat.causal) {  // per-head band launches of the same (maximal) band pair q-blocks
    AttnParams ph;
    build_schedule(B, Hq, Hkv, N, pat, num_ctas, true, &ph, false, true);
    *bytes = std::max(*bytes, ws_layout(ph, D).total);
  }
  return TM_OK;
}

int debug_schedule(int B, int Hq, int Hkv, int N, const Pattern& pat, int max_ctas, int split,
                   int qb_lo, int qb_hi, int* out, long long cap, long long* count, const int* hS,
                   const int* hW) {
  AttnParams p;
  const int grid = build_schedule(B, Hq, Hkv, N, pat, max_ctas, (split & 1) != 0, &p, false,
                                  (split & 2) != 0, qb_lo, qb_hi - qb_lo, hS, hW);
  long long n = 0;
  for (int c = 0; c < grid; ++c) {
    const int n_work = work_count(p, c, grid);
    for (int k = 0; k < n_work; ++k, ++n) {
      const Item it = work_item_at(p, c, grid, k);  // what the producer publishes
      const int item = work_item(p, c, grid, k);
      if (n >= cap) continue;
      const int T = item_tiles(p, it).count();
      int* r = out + 7 * n;
      // Q tiles: heads h0, h0 + 1 of q-block qb, or (q-block pairs, bit 8 set)
      // q-blocks qb, qb + 1 of head h0
      r[0] = c; r[1] = item; r[2] = it.qb; r[3] = it.b * Hq + it.h0;
      r[4] = 1 + it.v1 + (p.qpair ? 256 : 0);
      r[5] = it.t0; r[6] = std::min(T, it.t1);
    }
  }
  *count = n;
  return TM_OK;
}

int launch_dump_tiles(const Pattern& pat, int* out_dev, long long cap, void* stream) {
  const int nqb = (pat.N + BM - 1) / BM;
  if (cap <= 0) return TM_OK;
  dump_tiles_kernel<<<(nqb + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(pat, nqb,
                                                                                      out_dev, cap);
  return counted(1);
}

template <int D>
static int launch_probe_d(const void* q, const void* k, const void* v, float* s_out, float* o_out,
                          void* stream, DeviceInfo* di) {
  const int kidx = D == 128 ? 1 : 0;
  const int smem = 3 * Cfg<D>::kTileBytes + 64 + 1024;
  if (int rc = set_smem_once(di->probe_attr_set[kidx], mma_probe_kernel<D>, smem)) return rc;
  CUtensorMap tq, tk, tv;
  if (encode_bnhd(&tq, q, 1, 128, 1, D, 128) || encode_bnhd(&tk, k, 1, 128, 1, D, 128) ||
      encode_bnhd(&tv, v, 1, 128, 1, D, 128))
    return TM_ERR_CUDA;
  mma_probe_kernel<D><<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(tq, tk, tv, s_out,
                                                                          o_out);
  return counted(1);
}

int launch_mma_probe(const void* q, const void* k, const void* v, float* s_out, float* o_out,
                     int D, void* stream) {
  DeviceInfo* di = nullptr;
  if (int rc = device_info(&di)) return rc;
  if (D == 128) return launch_probe_d<128>(q, k, v, s_out, o_out, stream, di);
  if (D == 64) return launch_probe_d<64>(q, k, v, s_out, o_out, stream, di);
  return TM_ERR_UNSUPPORTED;
}

int read_and_clear_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TM_ERR_CUDA;
  int st = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&st, g_status, sizeof(int)) != cudaSuccess) return TM_ERR_CUDA;
  if (st != kDevOk) {
    int where = 0;
    cudaMemcpyFromSymbol(&where, g_status_where, sizeof(int));
    fprintf(stderr, "tm: kernel gave up on a pipeline wait (site %d)\n", where);
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return TM_ERR_CUDA;
    return TM_ERR_TIMEOUT;
  }
  return TM_OK;
}

}  // namespace trimix
