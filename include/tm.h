/*
 * tm.h - C ABI of the TriangleMix prefill-attention library for NVIDIA B200 (sm_100a).
 *
 * TriangleMix (He Zhiyuan's blog post "TriangleMix", sections 介绍 and 性能;
 * the 36kr interview with Yang Yuqing, lead paragraphs) runs dense causal
 * attention in the shallow layers of a model and a static "triangle" pattern
 * in the deep layers, from layer index tri_start on. In the triangle pattern
 * query row i attends key j (j <= i) only if
 *     j < S          (one of the first S "sink" tokens of the streaming region),
 *  or i - j < W      (one of the W most recent positions, i itself included),
 *  or i >= N - L     (i is one of the last L queries: the "last Q-K" region,
 *                     which sees every causal key).
 * Everything else (the "middle Q-K" region) is skipped. The result is exact
 * masked softmax attention over that key set:
 *     o_i = sum_{j in K_i} softmax_j(scale * q_i . k_j) v_j.
 *
 * Tensor layout (all entry points): bf16, contiguous,
 *     q, o : [B, N, Hq,  D]      k, v : [B, N, Hkv, D]
 * Query head hq reads kv head hq / (Hq / Hkv) (consecutive q heads share a kv
 * head). D must be 64 or 128. RoPE, if any, is applied by the caller.
 *
 * Numerics: scores and the softmax are fp32, the weights P bf16, and O, l fp32
 * sums on the tensor cores. The softmax reference (the running max) moves only
 * when a tile's scores exceed it by more than 48 in the log2 domain, so P stays
 * below 2^48. O stays finite for |v| up to about 2^62 over 2^17 keys, which is
 * far outside the range of activations.
 *
 * Ownership and threading:
 *   - q, k, v, o are DEVICE pointers owned by the caller, 16-byte aligned;
 *     o must not overlap q, k or v (tm_trianglemix_attn_fwd_host takes host
 *     buffers besides them). The library allocates no device memory in any
 *     call and keeps no per-call state; scratch for the split schedule is a
 *     caller-owned workspace (the *_ws calls). The host-buffer call creates
 *     two copy streams and a pool of events per device on first use and
 *     keeps them for the life of the process.
 *   - `stream` is a cudaStream_t (CUstream) handle passed as void*; NULL is
 *     the legacy default stream. Work is enqueued asynchronously on it and
 *     the call returns without synchronising.
 *   - Calls are thread-safe. No C++ exception crosses this interface.
 *
 * Errors: every entry point returns a tm_status. Argument errors are reported
 * synchronously, before anything is enqueued. TM_ERR_CUDA means a CUDA call
 * failed (launch or driver). A kernel that gives up waiting on one of its own
 * pipeline barriers (a bounded wait, about two seconds) records
 * TM_ERR_TIMEOUT in a device status word, finishes cleanly and leaves the
 * context usable; tm_get_device_status() reports it.
 */
#ifndef TM_H_
#define TM_H_

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define TM_API __declspec(dllexport)
#else
#define TM_API __attribute__((visibility("default")))
#endif

typedef enum {
  TM_OK = 0,
  TM_ERR_INVALID_ARG = -1,  /* null/misaligned/overlapping pointer, bad size or pattern */
  TM_ERR_UNSUPPORTED = -2,  /* valid but not built: D not in {64,128}, not an sm_100 device */
  TM_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed */
  TM_ERR_TIMEOUT = -4       /* a kernel gave up on a pipeline wait (device status) */
} tm_status;

/* Tile shape of the kernels (query rows x key columns per tile). */
#define TM_BLOCK_M 128
#define TM_BLOCK_N 128

/*
 * Dense causal attention, keep(i, j) = j <= i. This is the "full attention"
 * the TriangleMix pages compare against (blog post, section 速度).
 * scale: the softmax scale applied to q.k (commonly 1/sqrt(D)); must be finite and > 0
 *        (masked scores are -inf before scaling).
 */
TM_API int tm_causal_attn_fwd(const void* q, const void* k, const void* v, void* o, int B,
                              int Hq, int Hkv, int N, int D, float scale, void* stream);

/*
 * Triangle attention with sink count S, window W and last-query count L
 * (blog post, section 介绍 and the "Middle Q-K" figure discussion in 缘由;
 * 36kr interview, lead paragraph on the streaming and last Q-K regions).
 * S >= 0, L >= 0, W >= 1; S and L larger than N act as N. L = N, or S + W >= N,
 * gives the same result as tm_causal_attn_fwd.
 */
TM_API int tm_triangle_attn_fwd(const void* q, const void* k, const void* v, void* o, int B,
                                int Hq, int Hkv, int N, int D, float scale, int S, int W, int L,
                                void* stream);

/*
 * Layer schedule (blog post, section 性能: layers before the chosen start run
 * full attention, the rest run triangle attention; 36kr interview:
 * "L_tri_start = 12"). layer and tri_start are 0-based: layer < tri_start runs
 * tm_causal_attn_fwd, layer >= tri_start runs tm_triangle_attn_fwd with
 * (S, W, L). layer >= 0 and tri_start >= 0 are required; S, W, L are validated
 * only when the triangle kernel is chosen.
 */
TM_API int tm_trianglemix_attn_fwd(const void* q, const void* k, const void* v, void* o, int B,
                                   int Hq, int Hkv, int N, int D, float scale, int S, int W,
                                   int L, int layer, int tri_start, void* stream);

/*
 * The same layer call on HOST buffers, streamed: q_host, k_host, v_host are
 * read and o_host is written, in the [B, N, H, D] bf16 layout above.
 * - Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister); a
 *   pageable buffer still works, but its copies do not overlap.
 * - q_dev, k_dev, v_dev, o_dev: caller-owned device buffers of the same sizes
 *   and layout (16-byte aligned; o_dev overlapping none of the others), used
 *   as staging. The library allocates no device memory.
 * - The rows are taken in chunks of chunk_rows, a multiple of TM_BLOCK_M; 0
 *   picks 8192. Chunks grow so that there are at most 64.
 * - For chunk c, the library copies its q, k and v rows in on one internal
 *   stream, then computes its queries on `stream` as soon as they and every
 *   earlier chunk are resident, then copies its o rows out on a second
 *   internal stream. In causal order a chunk's queries need no later key, so
 *   copy-in, compute and copy-out of different chunks overlap.
 * - The result is bit for bit that of tm_trianglemix_attn_fwd on the same
 *   device buffers.
 * - Ordering: the copies start after the work queued on `stream` before the
 *   call, and `stream` completes only after the last copy-out. So the host
 *   buffers may be reused once `stream` has been synchronised. The call
 *   returns once all copies and kernels are queued.
 * - Calls on one device are enqueued one at a time (the internal streams are
 *   shared per device).
 * - Errors: TM_ERR_INVALID_ARG for a NULL host pointer or a bad chunk_rows,
 *   and otherwise as for tm_trianglemix_attn_fwd on the device buffers.
 *   TM_ERR_CUDA if a copy or launch cannot be queued; work queued before the
 *   failure still runs.
 */
TM_API int tm_trianglemix_attn_fwd_host(const void* q_host, const void* k_host,
                                        const void* v_host, void* o_host, void* q_dev,
                                        void* k_dev, void* v_dev, void* o_dev, int B, int Hq,
                                        int Hkv, int N, int D, float scale, int S, int W, int L,
                                        int layer, int tri_start, int chunk_rows, void* stream);

/*
 * Triangle attention with a band per q head: head h keeps the sinks j < S_h
 * and the window i - j < W_h, all heads share the last-L rows. This is the
 * bf16 reading of TriAttention's per-head regions (arXiv 2611.07256 abstract
 * on the TriAttention page: each head's computed region is encoded by two
 * diagonal-distance boundaries, independent of the context length); with both
 * precision regions computed in bf16 the computed region is one band below
 * the diagonal, here widened by the head's sinks.
 * S_heads, W_heads: HOST arrays of Hq ints (S_h >= 0, W_h >= 1; S_h and W_h
 * larger than N act as N); Hq <= 128. Each work item holds two consecutive
 * q-blocks of one head and visits the union of their tile lists, each Q tile
 * masked with its own rows, so a Q tile visits at most one tile it does not
 * need; the heads rotate across the CTAs. workspace / workspace_bytes
 * as for tm_triangle_attn_fwd_ws, sized by tm_attn_workspace_size with
 * S = max S_h and W = max W_h (NULL and 0 split nothing).
 */
TM_API int tm_triangle_attn_fwd_heads(const void* q, const void* k, const void* v, void* o, int B,
                                      int Hq, int Hkv, int N, int D, float scale,
                                      const int* S_heads, const int* W_heads, int L,
                                      void* workspace, long long workspace_bytes, void* stream);

/*
 * Block-sparse causal attention from a caller's block index, on the same
 * kernels: the visited tiles of each q-block come from the index instead of a
 * closed form, the way the FlashPrefill summary (section 2.3) jumps straight
 * to the selected blocks instead of testing every block. Meant for the
 * shallow layers that the TriangleMix blog post (section 介绍, last paragraph)
 * leaves to dynamic sparse methods; pattern discovery produces such an index.
 *   keep(i, j) = j <= i  and  j < N  and  j / TM_BLOCK_N is listed for
 *                (batch, kv head of the row's q head, q-block i / TM_BLOCK_M).
 * Index (DEVICE memory, int32, CSR): with nqb = ceil(N / TM_BLOCK_M) and
 * r = (b * Hkv + g) * nqb + qb, block_offsets[r] .. block_offsets[r + 1]
 * (B * Hkv * nqb + 1 entries, non-decreasing, within [0, nnz]) delimit the
 * k-blocks of that q-block in block_indices[0 .. nnz), which should be strictly
 * ascending in [0, qb]. All q heads of a kv head's group share its lists.
 * Offsets are clamped to [0, nnz] and entries outside [0, qb] are visited as
 * fully masked tiles, so a malformed index yields wrong values, never an
 * access outside q, k, v, o or the index; a duplicated entry counts its keys
 * twice. A row that keeps no key is written as zeros. The index is read by the
 * kernel (no host synchronisation).
 * tm_trianglemix_sparse_attn_fwd is the layer schedule with this as the
 * shallow layers: layer < tri_start runs the block-sparse call with the
 * index, layer >= tri_start runs tm_triangle_attn_fwd (the index is ignored).
 */
TM_API int tm_block_sparse_attn_fwd(const void* q, const void* k, const void* v, void* o, int B,
                                    int Hq, int Hkv, int N, int D, float scale,
                                    const int* block_offsets, const int* block_indices,
                                    long long nnz, void* stream);
TM_API int tm_trianglemix_sparse_attn_fwd(const void* q, const void* k, const void* v, void* o,
                                          int B, int Hq, int Hkv, int N, int D, float scale,
                                          int S, int W, int L, int layer, int tri_start,
                                          const int* block_offsets, const int* block_indices,
                                          long long nnz, void* stream);

/*
 * Block pattern discovery: builds the block index of tm_block_sparse_attn_fwd
 * on the GPU, after the FlashPrefill summary (section 2.1: uniformly spread
 * probe queries against average-pooled key blocks; section 2.2: keep the
 * blocks whose score reaches alpha times the best score of their query block,
 * no top-k / top-p sort). For batch b, kv head g and q-block I (rows
 * [r0, r1)):
 *   kbar_J       = mean of k[b, j, g, :] over the keys of block J
 *   probe rows   max(r0, r0 + ((p + 1) (r1 - r0)) / probes - 1), p = 0 .. probes-1,
 *                in each q head h of g's group
 *   pi_{h,p}(J)  = softmax over J in [0, I] of scale * q[b, row_p, h, :] . kbar_J
 *   Score(I, J)  = mean over (h, p) of pi_{h,p}(J)
 *   list(b,g,I)  = { J <= I : Score(I, J) >= alpha * max_J' Score(I, J') }, ascending
 * (the same q heads share each list, as tm_block_sparse_attn_fwd expects). The
 * pooled keys and probe rows are bf16 and the scores fp32 (tensor cores), so
 * a block whose score lies within rounding of the threshold may fall either
 * way. alpha in [0, 1] (0 keeps every causal block); 1 <= probes and
 * probes * (Hq / Hkv) <= 128; B * Hkv <= 65535.
 * Memory (all DEVICE, caller-owned): workspace of at least
 * tm_flashprefill_workspace_size bytes, 256-byte aligned; block_offsets of
 * B * Hkv * nqb + 1 ints; block_indices of cap >= tm_flashprefill_index_capacity
 * ints (the dense causal count, so a list never overflows); the number of
 * entries written is block_offsets[B * Hkv * nqb]. scores_out (optional, may
 * be NULL): B * Hkv * nqb * nqb floats receiving Score(I, J) at
 * ((b * Hkv + g) * nqb + I) * nqb + J for J <= I. Asynchronous on `stream`
 * (five launches, no host synchronisation).
 */
TM_API int tm_flashprefill_workspace_size(int B, int Hq, int Hkv, int N, int D, int probes,
                                          long long* bytes);
TM_API long long tm_flashprefill_index_capacity(int B, int Hkv, int N);
TM_API int tm_flashprefill_block_index(const void* q, const void* k, int B, int Hq, int Hkv, int N,
                                       int D, float scale, float alpha, int probes,
                                       void* workspace, long long workspace_bytes,
                                       int* block_offsets, int* block_indices, long long cap,
                                       float* scores_out, void* stream);

/*
 * Split schedule for the long q-blocks. The last L query rows of the triangle
 * (and the last rows of causal attention) see every earlier key, so one of
 * their items can cost more than a CTA's share of the launch when B * Hq is
 * small (a tensor-parallel shard, one sequence). With a workspace the
 * library cuts such items into pieces over ranges of their tile list; each
 * piece writes its unnormalised partial output with its running row max m and
 * row sum l, and the piece that finishes last merges them (log-sum-exp merge:
 * O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s) in piece
 * order, so the result is deterministic. The output equals that of the
 * entry points without a workspace up to float rounding.
 *
 * tm_attn_workspace_size: bytes of workspace the *_ws calls need for this
 * problem on a grid of num_ctas CTAs (pass 0 for the current device's SM
 * count); 0 if nothing would be split. Host only, except that num_ctas = 0
 * queries the device.
 *
 * tm_*_ws: the entry points above with a caller-owned DEVICE workspace of
 * workspace_bytes bytes, 16-byte aligned, not overlapping q, k, v or o.
 * workspace = NULL with workspace_bytes = 0 splits nothing (identical to the
 * calls without _ws). A workspace smaller than tm_attn_workspace_size reports
 * gives TM_ERR_INVALID_ARG. Each call clears the counters it uses (an async
 * memset on `stream`) and uses the rest as scratch: calls sharing one
 * workspace must be ordered (same stream, or synchronised); the contents are
 * undefined afterwards.
 */
TM_API int tm_attn_workspace_size(int B, int Hq, int Hkv, int N, int D, int causal, int S, int W,
                                  int L, int num_ctas, long long* bytes);
TM_API int tm_causal_attn_fwd_ws(const void* q, const void* k, const void* v, void* o, int B,
                                 int Hq, int Hkv, int N, int D, float scale, void* workspace,
                                 long long workspace_bytes, void* stream);
TM_API int tm_triangle_attn_fwd_ws(const void* q, const void* k, const void* v, void* o, int B,
                                   int Hq, int Hkv, int N, int D, float scale, int S, int W, int L,
                                   void* workspace, long long workspace_bytes, void* stream);
TM_API int tm_trianglemix_attn_fwd_ws(const void* q, const void* k, const void* v, void* o, int B,
                                      int Hq, int Hkv, int N, int D, float scale, int S, int W,
                                      int L, int layer, int tri_start, void* workspace,
                                      long long workspace_bytes, void* stream);

/*
 * tm_trianglemix_attn_fwd with the split schedule, for callers that cannot
 * hand the library device memory: the paper has no counterpart. Callers that
 * cannot allocate are, for instance, code running under a memory pool or a
 * framework that owns every device byte, or code on a path where an
 * allocation would synchronise the device. Instead of a caller workspace this
 * call uses a fixed scratch array of TM_NOALLOC_SCRATCH_BYTES (16 MiB) that
 * the library's module holds on every device that loads it, until the
 * process exits. The call allocates and frees nothing. The array's address is
 * looked up (cudaGetSymbolAddress) by the first call on each device context,
 * and again after that context is recreated; make the first call outside any
 * stream capture. A problem whose split needs more than the scratch (as
 * tm_attn_workspace_size reports on this device) runs the unsplit schedule
 * instead, which needs no scratch: the same attention, with the long items
 * not cut (its bits may differ from a split run's in the last place); so does
 * a problem with nothing to split. Each call that uses the scratch clears the
 * arrival counters it needs (an async memset on `stream`) before its kernel;
 * the rest of the array keeps the previous call's contents. Calls that
 * overlap in time on one device race on the scratch and give undefined
 * results: issue them on one stream, or order them otherwise.
 */
#define TM_NOALLOC_SCRATCH_BYTES (16LL << 20)
TM_API int tm_trianglemix_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                           int B, int Hq, int Hkv, int N, int D, float scale,
                                           int S, int W, int L, int layer, int tri_start,
                                           void* stream);

/*
 * Number of kept (i, j) pairs of one (batch, head) of the triangle pattern:
 * sum over rows of min(i+1, W) + max(0, min(S, i+1-W)) for i < N-L and i+1
 * otherwise. The kept set is the blog post's (TriangleMix blog post, section
 * 介绍): the sink and local parts of the streaming region for most rows, and
 * every causal key for the last L rows; the per-row closed form counts it with
 * the window including the diagonal and the sinks and window as a union.
 * Host only. Returns -1 on a bad argument.
 */
TM_API long long tm_triangle_kept_pairs(int N, int S, int W, int L);

/*
 * Number of TM_BLOCK_M x TM_BLOCK_N tiles the kernel visits for one
 * (batch, head): tiles holding at least one kept pair, the "kept tiles" whose
 * FLOPs the throughput counts. Only these tiles are visited, by index, rather
 * than branched over (FlashPrefill summary, section 2.3: physical jumps
 * instead of logical skipping). causal != 0 counts the causal pattern (S, W,
 * L ignored). Host only. -1 on a bad argument.
 */
TM_API long long tm_kept_tiles(int N, int causal, int S, int W, int L);

/*
 * Host export of the static tile list the kernels derive on the device, at
 * tile shape (BM, BN) (the kernels use TM_BLOCK_M x TM_BLOCK_N): the index by
 * which the kernels jump from kept tile to kept tile (FlashPrefill summary,
 * section 2.3), built from the triangle pattern's per-row kept intervals
 * (TriangleMix blog post, section 介绍). One record is
 * three ints (qb, kb, full): q-block, k-block, and 1 if every pair of the
 * tile's existing rows and columns is kept (no mask needed), else 0. Records
 * are ordered by qb ascending, then kb ascending; tiles without a kept pair
 * are absent. out: HOST buffer of 3*cap ints (may be NULL when cap = 0);
 * *count receives the total number of records even when it exceeds cap.
 * tm_triangle_tile_list is the triangle pattern; tm_tile_list selects causal.
 */
TM_API int tm_triangle_tile_list(int N, int S, int W, int L, int BM, int BN, int* out,
                                 long long cap, long long* count);
TM_API int tm_tile_list(int N, int causal, int S, int W, int L, int BM, int BN, int* out,
                        long long cap, long long* count);

/*
 * Device dump of the same list (FlashPrefill summary, section 2.3; TriangleMix
 * blog post, section 介绍), produced by the kernels' own device code at
 * TM_BLOCK_M x TM_BLOCK_N, so a test can compare what the device visits with
 * the host list bit for bit. Beyond the plain dump of the triangle list it
 * takes `causal` (the causal list, which the same device code produces) and
 * returns the record total in *count (host), so the caller can size the
 * buffer. out_dev: DEVICE buffer of 3*cap ints; records beyond cap are not
 * written. Asynchronous on `stream`.
 */
TM_API int tm_debug_dump_tiles(int N, int causal, int S, int W, int L, int* out_dev,
                               long long cap, long long* count, void* stream);

/*
 * Building-block check of the tensor-core path on one 128-row tile:
 * s_out[128*128] = q k^T (fp32) and o_out[128*D] = bf16(q k^T) v (fp32), with
 * q, k, v bf16 [128, D] DEVICE pointers and s_out, o_out fp32 DEVICE pointers.
 * Asynchronous on `stream`.
 */
TM_API int tm_debug_mma_probe(const void* q, const void* k, const void* v, float* s_out,
                              float* o_out, int D, void* stream);

/*
 * Host export of the persistent work split the kernels use on a grid of
 * num_ctas CTAs (the SM count on a B200). split: bit 0 gives the split
 * schedule of the *_ws calls (else the one of the calls without workspace),
 * bit 1 the item layout of per-head band launches (q-block pairs of one head
 * for non-causal patterns, and the rotations). One record of seven ints per
 * work item, (cta, item, q-block, first q head (batch * Hq + head), Q tiles,
 * first tile, end tile), in the order each CTA processes them; the tiles are
 * positions [first, end) in the item's tile list (the whole list unless the
 * item is a piece). An item covers one q-block of one or two q heads that
 * share a kv head; with q-block pairs (Q tiles has bit 8 set, 256 + 1 or 256 +
 * 2), one or two consecutive q-blocks of one head, whose tile list is the
 * union of theirs. Causal schedules of an odd group size (Hq / Hkv odd, above
 * 1) over all q-blocks use q-block pairs too. out: HOST buffer of 7*cap ints (NULL when cap = 0); *count
 * receives the total. Host only.
 */
TM_API int tm_debug_schedule(int B, int Hq, int Hkv, int N, int causal, int S, int W, int L,
                             int num_ctas, int split, int* out, long long cap, long long* count);

/*
 * tm_debug_schedule for the work of the q-blocks [qb_lo, qb_hi) only (qb_hi
 * -1: to the last q-block), the split that tm_trianglemix_attn_fwd_host runs
 * for one row chunk; q-block numbers in the records are global. Requires
 * 0 <= qb_lo < qb_hi <= ceil(N / TM_BLOCK_M). Host only.
 */
TM_API int tm_debug_schedule_window(int B, int Hq, int Hkv, int N, int causal, int S, int W,
                                    int L, int num_ctas, int split, int qb_lo, int qb_hi,
                                    int* out, long long cap, long long* count);

/*
 * tm_debug_schedule of a per-head band launch (tm_triangle_attn_fwd_heads)
 * with these bands: S_heads, W_heads are HOST arrays of Hq ints, as there.
 * The bands decide which CTAs sit out rounds for holding an extra heavy item.
 * Host only.
 */
TM_API int tm_debug_schedule_heads(int B, int Hq, int Hkv, int N, const int* S_heads,
                                   const int* W_heads, int L, int num_ctas, int split, int* out,
                                   long long cap, long long* count);

/*
 * Failure-detection check (tests only): runs tm_triangle_attn_fwd with one
 * fault injected on the host side of the pipeline — the producer of CTA 0
 * delivers no Q tile for its first item and stops. That CTA's MMA issuer then
 * gives up on its bounded wait (about two seconds), records TM_ERR_TIMEOUT in
 * the device status word, and all of the CTA's roles leave, drain their copies
 * and free TMEM; the other CTAs finish. o is left partly unwritten. The call
 * itself returns TM_OK (or an argument error); tm_get_device_status then
 * reports TM_ERR_TIMEOUT, and the context stays usable.
 */
TM_API int tm_debug_inject_stall(const void* q, const void* k, const void* v, void* o, int B,
                                 int Hq, int Hkv, int N, int D, float scale, int S, int W, int L,
                                 void* stream);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device: TM_OK, or TM_ERR_TIMEOUT if a kernel gave up on a wait
 * since the last call. TM_ERR_CUDA if the synchronisation itself failed.
 */
TM_API int tm_get_device_status(void* stream);

/* Static string for a status code; never NULL. */
TM_API const char* tm_status_string(int status);

/*
 * Number of kernels this library has launched in the calling process so far
 * (every launch whose enqueue succeeded, on any device and stream; the
 * host-buffer call's copies are not kernels and do not count). Read it
 * before and after a region to count the library's launches inside it; the
 * paper has no counterpart: it is measurement support. Host only, never
 * fails.
 */
TM_API long long tm_debug_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* TM_H_ */
