/*
 * mala.h - C ABI of the B200 (sm_100a) MassAlloc Attention (MALA) library.
 *
 * MALA is causal softmax attention that computes every legal causal QK^T score tile
 * and then runs the post-score work of a tile (exp, P.V and, in backward, the
 * dP/dS/dQ/dK/dV products) only when the tile's normalised contribution reaches the
 * length-normalised tolerance tau / L_q.  Source: "MassAlloc Attention: Let Attention
 * Allocate Its Own Compute" (§2.1 tolerance, §2.2 Eq. (3) online forward test and
 * Eq. (4) offline backward test, §2.4 split-KV decoding, App. A Algorithms 1 and 2).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are caller-owned DEVICE memory, contiguous, 16-byte aligned.
 *   - Layouts: Q, O, dO, dQ [B, L, H, d]; K, V, dK, dV [B, L, H_kv, d];
 *     LSE [B, H, L] float32, natural-log log-sum-exp of the scaled scores over the
 *     retained keys (the page's final l = m + log l).  Query head h reads KV head
 *     h / (H / H_kv) (grouped-query attention).
 *   - Scores are s = scale * <q, k>; tiles are 128 query rows x 128 keys; tile (i, j)
 *     is query block i, key block j.  The forward visits j = i, i-1, ..., 0 (diagonal
 *     first) and skips a tile only when every valid row with a legal key in it has
 *     max_k s - log Z_q < log(tau / L_q), L_q = q + 1 (strict; ties retain).
 *   - tau >= 0.  tau == 0 means "never skip" and runs the same library's dense
 *     FlashAttention-style kernels; MALA_FLAG_ALWAYS_TEST runs the retention test
 *     anyway (it then retains everything) to measure its overhead.
 *   - dtype: MALA_BF16 (tensor-core path; d in {64, 128}) or MALA_FP32 (fp32 SIMT path
 *     for small problems; d <= 128).
 *   - tile_mask (optional, may be NULL): debug output of the decisions, one byte per
 *     legal tile, 1 = retained, 0 = skipped.  Forward / backward: [B, H, T, T] with
 *     T = ceil(L / 128), entry [b][h][i][j]; decode: [B, H, T] with T = ceil(N_k / 128).
 *     Entries of illegal tiles (j > i) are left untouched.  The method itself never
 *     materialises a mask; this buffer exists only for testing and statistics.
 *   - workspace: caller-provided device scratch of at least the size returned by the
 *     matching *_workspace_bytes query.  Passing workspace == NULL makes the library
 *     allocate it stream-ordered (cudaMallocAsync / cudaFreeAsync) on `stream`.  The
 *     first 256 bytes of any workspace hold counters and the device error word.
 *   - stream: a cudaStream_t (NULL = legacy default stream).  All work is enqueued
 *     asynchronously; no entry point synchronises the host.
 *   - Errors: arguments are validated before anything is launched
 *     (MALA_ERR_INVALID_ARG / MALA_ERR_UNSUPPORTED); launch failures return
 *     MALA_ERR_CUDA.  A kernel whose internal wait runs out of its time budget records
 *     MALA_ERR_TIMEOUT in the workspace error word and returns early instead of
 *     hanging; read it with mala_read_device_error().
 */
#ifndef MALA_H
#define MALA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MALA_OK = 0,
  MALA_ERR_INVALID_ARG = 1,
  MALA_ERR_UNSUPPORTED = 2,
  MALA_ERR_CUDA = 3,
  MALA_ERR_TIMEOUT = 4,
  MALA_ERR_WORKSPACE = 5
} mala_status;

typedef enum { MALA_BF16 = 0, MALA_FP32 = 1 } mala_dtype;

/* flags */
#define MALA_FLAG_ALWAYS_TEST 1u /* evaluate the retention test even when tau == 0 */

/*
 * mala_fwd - MALA forward (training forward and inference prefill).
 * "MassAlloc Attention", §2.2 (online sparse softmax, Eq. (1)-(3)), App. A Algorithm 1
 * and A.1 (fused forward execution).
 *   Q [B,L,H,d], K/V [B,L,H_kv,d] in, O [B,L,H,d] out (same dtype as the inputs),
 *   LSE [B,H,L] float32 out.  Causal, N_q = N_k = L >= 1.
 */
mala_status mala_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                     int H, int H_kv, int L, int d, int dtype, float scale, float tau,
                     unsigned flags, void* workspace, size_t workspace_bytes,
                     uint8_t* tile_mask, void* stream);

/*
 * mala_fwd_prefill - MALA forward of a prefill chunk (chunked prefill).
 * "MassAlloc Attention", §2.3 (the same forward serves inference prefill) with the
 * forward rules of §2.2 / Algorithm 1.  The N_q queries are the last N_q positions of a
 * sequence of N_k >= N_q keys that already holds them (the KV cache including the chunk):
 * query row q sits at position p = N_k - N_q + q, attends to keys k <= p, and is tested
 * with L_q = p + 1.  Query block i (rows [128 i, 128 i + 128)) visits the key blocks that
 * hold a legal key of one of its rows, from the last one down to 0; when N_k - N_q is not
 * a multiple of 128 the block straddles two key blocks, and both are masked per row.
 *   Q [B,N_q,H,d], K/V [B,N_k,H_kv,d] in; O [B,N_q,H,d], LSE [B,H,N_q] float32 out.
 *   tile_mask (optional) is [B, H, ceil(N_q/128), ceil(N_k/128)], entry [b][h][i][j].
 *   N_q == N_k is exactly mala_fwd.  Workspace: mala_fwd_workspace_bytes(B,H,H_kv,N_q,d,.).
 *   Errors as mala_fwd; N_q > N_k is MALA_ERR_INVALID_ARG.
 */
mala_status mala_fwd_prefill(const void* Q, const void* K, const void* V, void* O, float* LSE,
                             int B, int H, int H_kv, int N_q, int N_k, int d, int dtype,
                             float scale, float tau, unsigned flags, void* workspace,
                             size_t workspace_bytes, uint8_t* tile_mask, void* stream);

/*
 * mala_fwd_varlen - MALA forward of a packed batch of sequences of different lengths.
 * "MassAlloc Attention", §2.3 (the forward serves inference prefill) with the rules of
 * mala_fwd_prefill applied to each sequence on its own.
 *   Sequence s owns query rows [cu_seqlens_q[s], cu_seqlens_q[s+1]) of Q / O and key
 *   rows [cu_seqlens_k[s], cu_seqlens_k[s+1]) of K / V; its N_q,s queries are the last
 *   N_q,s of its N_k,s >= N_q,s positions (N_q,s == N_k,s: a full causal sequence; a
 *   sequence may have N_q,s == 0).
 *   Q, O [total_q, H, d]; K, V [total_k, H_kv, d] (bf16, d in {64, 128}); LSE [H, total_q]
 *   float32.  cu_seqlens_q / cu_seqlens_k are HOST arrays of n_seqs + 1 non-decreasing
 *   offsets starting at 0.
 *   The workspace is required (mala_fwd_varlen_workspace_bytes): it receives a table of
 *   the batch's (sequence, query block) units, heaviest first, copied from host memory
 *   with cudaMemcpyAsync, so the call waits for earlier work on `stream` before it
 *   returns (pageable staging) and cannot be captured in a CUDA graph.  No tile_mask;
 *   mala_get_stats reports the call's tiles.  Each sequence's results equal those of
 *   mala_fwd_prefill on that sequence alone.  A batch with no query rows at all returns
 *   MALA_OK after the host checks, with no CUDA call (the workspace, statistics included,
 *   is left as it was).
 */
size_t mala_fwd_varlen_workspace_bytes(const int* cu_seqlens_q, int n_seqs, int H, int H_kv,
                                       int d, int dtype);
mala_status mala_fwd_varlen(const void* Q, const void* K, const void* V, void* O, float* LSE,
                            const int* cu_seqlens_q, const int* cu_seqlens_k, int n_seqs, int H,
                            int H_kv, int d, int dtype, float scale, float tau, unsigned flags,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * mala_bwd - MALA backward.
 * "MassAlloc Attention", §2.2 (offline sparse probability, Eq. (4)), App. A
 * Algorithm 2 and A.1 (fused backward execution).  O and LSE are the forward's
 * outputs; D = rowsum(O * dO) is formed inside.  dQ, dK, dV are fully written (not
 * accumulated); dK / dV sum the contributions of the H / H_kv query heads of each KV
 * head.  The workspace holds a float32 dQ accumulator [B,L,H,d] and D [B,H,L]; for
 * bf16 problems with few work units (B * H_kv * (L/128 + 1) below 592, e.g. one KV head
 * up to 64K tokens) it also holds float32 dK and dV accumulators [B,L,H_kv,d]: the query
 * heads of a KV head are then split over several CTAs, which add their dK / dV shares.
 * mala_bwd_workspace_bytes accounts for all of it.
 */
mala_status mala_bwd(const void* Q, const void* K, const void* V, const void* O,
                     const float* LSE, const void* dO, void* dQ, void* dK, void* dV, int B,
                     int H, int H_kv, int L, int d, int dtype, float scale, float tau,
                     unsigned flags, void* workspace, size_t workspace_bytes,
                     uint8_t* tile_mask, void* stream);

/*
 * mala_decode - MALA split-KV decoding of one query token per sequence.
 * "MassAlloc Attention", §2.1 (L_0 = N_k, including the current token), §2.4 and A.1
 * (each split tests against its own partial normaliser; splits merged by the
 * normaliser-aware log-sum-exp reduction).
 *   q [B,H,d]; Kc, Vc [B,N_k,H_kv,d] (the cache already holds the current token at
 *   position N_k - 1); O [B,H,d] out; LSE [B,H] float32 out.
 *   Key tiles of 128; split s of S owns tiles [s*T/S, (s+1)*T/S) (integer division)
 *   and visits them newest first.  num_splits = 0 picks mala_decode_num_splits().
 *   The bf16 path takes groups of up to 8 query heads per KV head (H / H_kv <= 8, else
 *   MALA_ERR_UNSUPPORTED); the fp32 path takes any group.
 *   The retained support depends on the split count (the page says so).
 */
mala_status mala_decode(const void* q, const void* Kc, const void* Vc, void* O, float* LSE,
                        int B, int H, int H_kv, int Nk, int d, int dtype, float scale,
                        float tau, int num_splits, unsigned flags, void* workspace,
                        size_t workspace_bytes, uint8_t* tile_mask, void* stream);

/*
 * mala_decode_noalloc - mala_decode for callers that cannot allocate device memory.
 * The attention page has no counterpart to this entry point; it exists for runtimes
 * that forbid allocation on their hot path (a fixed memory plan after warm-up, a plugin
 * inside a framework that owns the device allocator, code that must not call
 * cudaMalloc or cudaMallocAsync per call).
 *   Same arguments and results as mala_decode without the workspace: the scratch comes
 *   from a fixed array of MALA_DECODE_NOALLOC_SCRATCH_BYTES compiled into the library,
 *   which every GPU that loads the library holds until the process exits.  Calls whose
 *   mala_decode_workspace_bytes() exceeds that size return MALA_ERR_WORKSPACE.  With
 *   num_splits = 0 the split rule keeps B * H_kv * S <= 296 whenever B * H_kv <= 296, so
 *   the scratch is at most 296 * (H / H_kv) * (d + 1) * 4 bytes plus a small header:
 *   every bf16 decode (groups of up to 8) of such a batch fits.
 *   The first call on a device looks up the array's device address (once per device and
 *   driver context, with that device current; again after the context was recreated, e.g.
 *   by cudaDeviceReset); make that first call before any stream capture.
 *   All calls on a device share the array: calls whose work overlaps on the GPU (two
 *   streams at once) race and must be serialised by the caller.  Device-side wait
 *   timeouts are recorded in the internal array and are not reported by this call.
 */
#define MALA_DECODE_NOALLOC_SCRATCH_BYTES (4u << 20)
mala_status mala_decode_noalloc(const void* q, const void* Kc, const void* Vc, void* O,
                                float* LSE, int B, int H, int H_kv, int Nk, int d, int dtype,
                                float scale, float tau, int num_splits, unsigned flags,
                                uint8_t* tile_mask, void* stream);

/*
 * mala_get_stats - work statistics of the last call that ran on `workspace`.
 * The attention page reports the retained fraction of post-score work (§3); these counters
 * give it without a tile_mask buffer.  Every call that receives a caller workspace zeroes
 * them first and its kernels add to them (the fp32 forward, which needs no workspace,
 * fills them when one is passed anyway).  Synchronises `stream`.
 *   Forward / backward: legal_tiles = causal tiles tested, one per (b, h, i, j);
 *   retained_tiles = tiles whose post-score work ran; v_tiles_loaded = 0.
 *   Decode: legal_tiles = (b, h, key tile) pairs tested; retained_tiles = pairs retained;
 *   v_tiles_loaded = V tiles fetched (one per (b, KV head, tile) that some head of the
 *   group retains; per (b, h) on the fp32 path).
 * Calls made with workspace == NULL, and mala_decode_noalloc, keep no statistics.
 */
typedef struct {
  uint64_t legal_tiles;
  uint64_t retained_tiles;
  uint64_t v_tiles_loaded;
} mala_stats;
mala_status mala_get_stats(const void* workspace, void* stream, mala_stats* out);

/* Workspace sizes (bytes) for the calls above; 0 on invalid arguments. */
size_t mala_fwd_workspace_bytes(int B, int H, int H_kv, int L, int d, int dtype);
size_t mala_bwd_workspace_bytes(int B, int H, int H_kv, int L, int d, int dtype);
size_t mala_decode_workspace_bytes(int B, int H, int H_kv, int Nk, int d, int dtype,
                                   int num_splits);

/* The split count used when mala_decode is given num_splits = 0 (deterministic, host
 * only, no device query).  Among the counts that give at most two waves of units
 * (b, KV head, split) over 148 persistent CTAs, it takes the S that minimises
 * waves x (ceil(T / S) + 10) + S / 9: a CTA's time is its key tiles plus a fixed cost of
 * about ten tiles per unit, and merging the S partials of a (b, KV head) costs about
 * S / 9 tiles.  Ties go to fewer splits.  Returns 0 for invalid shapes. */
int mala_decode_num_splits(int B, int H, int H_kv, int Nk);

/* Reads the device error word of a workspace (synchronises `stream`).  *out receives
 * 0 or a mala_status code in its low byte (upper bits: which wait gave up).  Clears
 * the word when clear != 0. */
mala_status mala_read_device_error(const void* workspace, void* stream, uint32_t* out,
                                   int clear);

/*
 * mala_selftest_wait_timeout - test hook for the failure handling of the kernels' waits
 * (the page has no counterpart).  Launches one CTA whose single thread waits on an
 * mbarrier that nothing ever arrives on, using the same bounded wait as the kernels
 * (wall-clock budget budget_ns, 1 ns .. 10 s).  The wait runs out and records
 * MALA_ERR_TIMEOUT (low byte; upper bits name the wait) in the workspace error word, which
 * this call zeroes first; read it with mala_read_device_error().  No fault, trap or hang:
 * the kernel returns and the context stays usable.
 */
mala_status mala_selftest_wait_timeout(void* workspace, uint64_t budget_ns, void* stream);

/* Sets the wall-clock budget of every internal wait (default 2 s; test hook). */
mala_status mala_set_wait_budget_ns(uint64_t ns);

/*
 * mala_set_debug - test hook that exports the margin of every retention test.
 * The decisions are the threshold tests of "MassAlloc Attention" §2.2 Eq. (3) (forward),
 * Eq. (4) (backward) and §2.4 (decode); this hook reports how far each tested tile was
 * from its threshold, so that a caller can compare the decisions against an independent
 * evaluation and see how close a disagreeing tile was.  The page has no API for it.
 *   dbg->tile_margin: DEVICE float32 buffer with the layout of the call's tile_mask
 *   ([B,H,T,Tk] for mala_fwd / mala_fwd_prefill, [B,H,T,T] for mala_bwd, [B,H,T] for
 *   mala_decode); dbg->tile_margin_count: floats available in it.  Passing NULL, or a
 *   NULL tile_margin, turns the hook off.  The setting belongs to the calling host
 *   thread and stays until changed; mala_fwd_varlen and mala_decode_noalloc ignore it.
 *   A call that needs more entries than tile_margin_count returns MALA_ERR_INVALID_ARG
 *   before anything is launched.
 *   Each call first fills its entries with the all-ones bit pattern (a NaN) and then
 *   writes, for every tile whose test ran, the margin in natural-log units:
 *     forward: max over the block's rows with a legal key of
 *              max_k s_qk - log Z_q - log(tau / L_q), Z_q the running normaliser of the
 *              tiles retained so far, +inf if some such row has Z_q = 0;
 *     backward: max over the tile's legal entries of s_qk - LSE_q - log(tau / L_q);
 *     decode:  max_k s_k - log Z - log(tau / N_k) per head, Z the split's running
 *              normaliser, +inf on the first tile of a split.
 *   The tile is retained exactly when its margin is >= 0.  Margins are written only when
 *   the test runs (tau > 0 or MALA_FLAG_ALWAYS_TEST); other entries stay NaN.  The
 *   kernels combine the forward and backward margins with float atomics, so a call with
 *   the hook on runs slower.
 */
typedef struct {
  float* tile_margin;
  size_t tile_margin_count;
} mala_debug;
mala_status mala_set_debug(const mala_debug* dbg);

const char* mala_status_string(mala_status s);

/* Library version: 203 = 0.2.3 (0.2.0 added mala_fwd_prefill, mala_fwd_varlen and
 * mala_get_stats; 0.2.1 changes the automatic decode split count, mala_decode_num_splits;
 * 0.2.2 adds mala_set_debug; 0.2.3 changes the automatic decode split count again, for
 * small batches: it now accounts for the cost of merging the splits). */
int mala_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MALA_H */
