/*
 * adamas.h -- C ABI of the B200 (sm_100a) ADAMAS sparse decode attention library.
 *
 * The method is the one described in the ADAMAS long-context sparse attention
 * article (lnwmold.com/news/826806):
 *   §2.1  queries and cached keys are rotated by an orthogonal Hadamard matrix,
 *         which leaves every q.k unchanged and spreads outlier channels;
 *   §2.2  each rotated vector is bucketed into 2-bit codes by three dynamic
 *         thresholds (-m/2, 0, +m/2), m = max |y| over the 128-dim group;
 *   §3.1  the codes are kept as a packed cache, four codes per byte;
 *   §2.3  every cached token is scored by the Manhattan (L1) distance between
 *         its codes and the query's codes (a smaller distance is more relevant);
 *   §5.2  only a token budget of the best-scoring tokens is kept, and exact
 *         softmax attention runs over the K/V rows of those tokens.
 *
 * Conventions shared by every entry point
 *   - Head dimension d must be 128 (one bucketing group per vector).
 *   - Tensors are dense row-major in device memory:
 *       q       [B][Hq][128]          bf16
 *       K, V    [B][Hkv][Nmax][128]   bf16
 *       codes   [B][Hkv][Nmax][32]    uint8, four 2-bit codes per byte, the code of
 *                                     dimension 4j in bits 7:6 of byte j
 *       out     [B][Hq][128]          fp32
 *       idx     [B][Hq][budget]       int32
 *     Query head h reads kv head h / (Hq / Hkv) (grouped-query attention).
 *   - The caller owns every buffer and the stream.  Calls only enqueue work on
 *     `stream` (a cudaStream_t; NULL is the legacy default stream) and return;
 *     they never allocate, free or synchronise, except adamas_get_device_error,
 *     which synchronises `stream` to read the error word.
 *   - codes must be 32-byte aligned (it is streamed with 32-byte loads); the
 *     other bf16/fp32 tensors and the workspace 16-byte aligned; int32 arrays
 *     4-byte aligned.  Inputs must be finite: NaN or Inf in q or K gives
 *     unspecified codes, indices and outputs (never an out-of-bounds access).
 *   - Argument errors are detected on the host before anything is enqueued and
 *     are returned as a negative status; nothing is written in that case.  A
 *     failed launch returns ADAMAS_ERR_CUDA.  Conditions only the GPU can see
 *     (a sequence length outside [0, Nmax], a cross-block wait that timed out)
 *     set bits of an error word in the workspace; see adamas_get_device_error.
 *   - No exception crosses this interface.  All entry points are thread-safe
 *     for distinct workspaces.
 */
#ifndef ADAMAS_H
#define ADAMAS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without including the CUDA runtime headers */
typedef struct CUstream_st *adamas_stream_t;

enum adamas_status {
    ADAMAS_OK = 0,
    ADAMAS_ERR_INVALID_ARG = -1, /* null/misaligned pointer, bad size or shape */
    ADAMAS_ERR_UNSUPPORTED = -2, /* d != 128, group size > 8, batch > 1024, ... */
    ADAMAS_ERR_WORKSPACE = -3,   /* workspace missing or smaller than adamas_workspace_bytes */
    ADAMAS_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed */
    ADAMAS_ERR_DEVICE = -5       /* the device error word is non-zero */
};

/* Bits of the device error word. */
#define ADAMAS_DEVERR_SEQLEN 0x1u  /* a seq_lens entry was outside [0, Nmax]; it was clamped */
#define ADAMAS_DEVERR_TIMEOUT 0x2u /* a bounded wait on a stage copy gave up; the step's outputs are invalid */
#define ADAMAS_DEVERR_INTERNAL 0x4u /* a block's share exceeded its planned size; outputs are invalid */
#define ADAMAS_DEVERR_TABLE 0x8u    /* a block-table entry was outside [0, n_pages); page 0 was read instead */

/* Selection policies of adamas_decode_step_ex. */
enum adamas_select_policy {
    ADAMAS_SELECT_PER_HEAD = 0,    /* every query head keeps its own budget of tokens */
    ADAMAS_SELECT_GROUP_SHARED = 1 /* one budget per kv head, ranked by the distance summed over its query heads */
};

/* Static description of a status code (never NULL). */
const char *adamas_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int adamas_version(void);

/* Text of the last CUDA error that made a call of this thread return
 * ADAMAS_ERR_CUDA ("no CUDA error" if none).  Never NULL. */
const char *adamas_last_error_string(void);

/*
 * Bytes of device workspace adamas_decode_step needs for these sizes on the
 * current CUDA device (0 when the sizes are unsupported).  The workspace holds
 * the device error word and, only when a block's token distances do not fit in
 * shared memory (very long contexts), a spill area for them; histograms and
 * partial softmax states stay on chip.  For long contexts over few kv heads
 * (fewer clusters than fill 3/4 of the SMs, at least 65,536 tokens) the step
 * splits every (b, kv head) into slices inside the GPU, and the workspace also
 * carries the slices' histograms and softmax states.  It must be zero-filled once
 * before its first use (adamas_workspace_init); every step leaves it ready for the
 * next one.  One workspace must not be used by two steps that may run
 * concurrently.
 */
size_t adamas_workspace_bytes(int B, int Hq, int Hkv, int64_t Nmax, int d, int budget);

/* Zero-fill a workspace on `stream` (asynchronous).  Also the way to clear the
 * error word and recover after ADAMAS_DEVERR_TIMEOUT. */
int adamas_workspace_init(void *workspace, size_t workspace_bytes, adamas_stream_t stream);

/*
 * Encode cached keys into packed 2-bit codes (article §2.1 rotation, §2.2
 * bucketing, §3.1 packing).  For every (b, kv head) it encodes positions
 * [p, p + count) with p = pos_begin[b] (pos_begin: device int32[B], or NULL for
 * p = 0); positions outside [0, Nmax) are skipped.  Use count = Nmax at prefill
 * and count = 1 with pos_begin = the new token's position when appending.
 *   K      device bf16 [B][Hkv][Nmax][128]  (read)
 *   codes  device uint8 [B][Hkv][Nmax][32]  (written at the encoded positions)
 * The rotation is an fp32 Sylvester-order butterfly (stage widths 1..64, no
 * fused multiply-add) followed by one multiply by RN(1/sqrt(128)); the codes are
 * bit-identical to the CPU oracle's.
 */
int adamas_encode_keys(const void *K, uint8_t *codes, const int32_t *pos_begin, int count, int B,
                       int Hkv, int64_t Nmax, int d, adamas_stream_t stream);

/*
 * One decode step of one attention layer for the whole batch: encode q, score
 * every cached token t < seq_lens[b] of the query head's kv head by the L1
 * distance D of the codes (article §2.3), keep k_eff = min(budget, seq_lens[b])
 * tokens of smallest (D, t) -- ties go to the lower token index -- and run exact
 * softmax attention with scale 1/sqrt(128) over their bf16 K/V rows, in fp32.
 *   q         device bf16 [B][Hq][128]
 *   codes     device uint8 [B][Hkv][Nmax][32]  (from adamas_encode_keys)
 *   K, V      device bf16 [B][Hkv][Nmax][128]
 *   seq_lens  device int32 [B]
 *   out       device fp32 [B][Hq][128]   softmax-weighted sum of the kept V rows
 *                                        (0 when k_eff = 0)
 *   idx       device int32 [B][Hq][budget]  kept token positions in (D, t)
 *                                        order, -1 past k_eff
 *   workspace device, >= adamas_workspace_bytes(...) bytes, zero-filled once
 * The step runs as one kernel launch: one thread-block cluster per (b, kv head),
 * its blocks splitting the head's tokens and exchanging histograms and partial
 * softmax states through distributed shared memory.  The launch opts in to
 * programmatic dependent launch: its blocks may be scheduled while the previous
 * kernel of the stream drains, and each waits for that kernel to complete (and
 * its writes to be visible) before its first global read or write, so stream
 * order semantics are unchanged.
 */
int adamas_decode_step(const void *q, const uint8_t *codes, const void *K, const void *V,
                       const int32_t *seq_lens, int B, int Hq, int Hkv, int64_t Nmax, int d,
                       int budget, float *out, int32_t *idx, void *workspace,
                       size_t workspace_bytes, adamas_stream_t stream);

/*
 * adamas_encode_keys for one appended token per sequence followed by
 * adamas_decode_step, in one launch -- the usual decode-loop step (article §3.1:
 * the code cache grows by one row per generated token; §2.3, §5.2: the step then
 * scores and selects over the whole cache).  For every (b, kv head) with
 * 0 <= append_pos[b] < Nmax, the key K[b][kvh][append_pos[b]] (already written by
 * the caller) is encoded into codes exactly as adamas_encode_keys would, before
 * the step scores that position; other values of append_pos[b] append nothing.
 *   codes       device uint8 [B][Hkv][Nmax][32], read and written
 *   append_pos  device int32 [B]
 * Every other argument, result and rule is adamas_decode_step's; the results are
 * bit-identical to adamas_encode_keys(count 1, pos_begin = append_pos) followed
 * by adamas_decode_step.
 */
int adamas_decode_step_append(const void *q, uint8_t *codes, const void *K, const void *V,
                              const int32_t *seq_lens, const int32_t *append_pos, int B, int Hq,
                              int Hkv, int64_t Nmax, int d, int budget, float *out, int32_t *idx,
                              void *workspace, size_t workspace_bytes, adamas_stream_t stream);

/*
 * Debug and test entry point: the distances the decode step ranks by.
 *   dist  device uint16 [B][Hq][Nmax]: D in [0, 384] for t < seq_lens[b],
 *         0xFFFF past the sequence length.
 * Same argument rules as adamas_decode_step; seq_lens outside [0, Nmax] are
 * clamped (no error word here).
 */
int adamas_score(const void *q, const uint8_t *codes, const int32_t *seq_lens, int B, int Hq,
                 int Hkv, int64_t Nmax, int d, uint16_t *dist, adamas_stream_t stream);

/*
 * adamas_decode_step for callers that cannot allocate device memory where they
 * decode -- an allocator that must not be re-entered from the decode loop, a hook
 * that runs with allocation forbidden, or a program that only receives pointers
 * to memory someone else owns.  The ADAMAS article has no counterpart of this
 * entry point; it is a property of this library.
 *
 * Same arguments, results and rules as adamas_decode_step, without the
 * workspace: the scratch is a fixed 4 MiB array that the library keeps in the
 * global memory of every device it is loaded on, until the process exits.
 * Nothing is allocated or freed by this call.
 *   - Sizes whose workspace (adamas_workspace_bytes) exceeds 4 MiB are rejected
 *     with ADAMAS_ERR_WORKSPACE before anything is enqueued; use
 *     adamas_decode_step for those.
 *   - Every call on a device shares the one array, and it keeps the previous
 *     call's contents.  The call clears what must start at zero, but calls that
 *     may overlap on the GPU (different streams, or different threads without
 *     ordering) race on it; serialise them.
 *   - The device error word lives in the shared array; every call clears it
 *     first.  adamas_static_device_error reads the last call's word.
 *   - The array's address is looked up once per CUDA context (keyed by the
 *     context's process-unique id) and cached.  cudaDeviceReset destroys the
 *     context and the array's contents with it; the next call, in the new
 *     context, looks the address up again.
 */
int adamas_decode_step_static(const void *q, const uint8_t *codes, const void *K, const void *V,
                              const int32_t *seq_lens, int B, int Hq, int Hkv, int64_t Nmax, int d,
                              int budget, float *out, int32_t *idx, adamas_stream_t stream);

/*
 * Reads the device error word of the last adamas_decode_step_static call on the
 * current device (the word lives in the fixed scratch array; see
 * adamas_get_device_error for its bits).  Synchronises `stream`, so call it on
 * the stream of the decode calls, after them.  The word stays until the next
 * static call clears it.
 * Returns ADAMAS_OK when the word is 0, ADAMAS_ERR_DEVICE when a bit is set
 * (*error_word holds them), ADAMAS_ERR_INVALID_ARG for a NULL error_word,
 * ADAMAS_ERR_CUDA when the copy fails.
 */
int adamas_static_device_error(uint32_t *error_word, adamas_stream_t stream);

/*
 * Every option of the decode step in one call.  adamas_decode_step and
 * adamas_decode_step_append are this call with the optional fields zero.
 *
 * Required fields (as in adamas_decode_step):
 *   q, codes, K, V, seq_lens, B, Hq, Hkv, Nmax, d, budget, out, idx,
 *   workspace, workspace_bytes
 *
 * Optional fields (zero / NULL: off):
 *   append_pos   device int32 [B]: the key at append_pos[b] is encoded into codes
 *                before the step scores it (adamas_decode_step_append; the ADAMAS
 *                article's §3.1: the code cache grows by one row per token).
 *   k_new, v_new device bf16 [B][Hkv][128], both or neither, only with append_pos:
 *                the launch itself writes these rows into K and V at append_pos[b]
 *                (and encodes k_new), so a decode loop needs no separate copy of the
 *                new token's rows into the cache.  K and V are written.
 *   block_table  device int32 [B][max_pages]: a paged cache.  Token t of sequence b
 *                lives in physical page block_table[b][t / page_size] at slot
 *                t % page_size; codes, K and V are then page arrays laid out
 *                [n_pages][Hkv][page_size][32 or 128] (every kv head's rows of a page
 *                contiguous), and Nmax is ignored (max_pages * page_size tokens per
 *                sequence).  adamas_encode_keys encodes such a cache as B = n_pages
 *                sequences of Nmax = page_size tokens.  An entry outside
 *                [0, n_pages) sets ADAMAS_DEVERR_TABLE (the step then reads page 0).
 *                Requires n_pages * Hkv * page_size <= 2^31 - 1.
 *   page_size, max_pages, n_pages   the paged cache's geometry.
 *   n_sink, n_recent  forced rows: the first n_sink and the last n_recent tokens of
 *                every sequence rank ahead of every scored token (in index order), as
 *                attention sinks and a recent window; the rest are ranked by (D, t).
 *                When they outnumber k_eff the lowest indices win.
 *   policy       ADAMAS_SELECT_PER_HEAD (default) or ADAMAS_SELECT_GROUP_SHARED: for
 *                every (b, kv head) the distances of its G query heads are summed per
 *                token, k_eff tokens of smallest (sum, t) are kept once, and every
 *                query head of the group attends over them; idx is then
 *                [B][Hkv][budget] and budget must be <= 4096 (ADAMAS_ERR_UNSUPPORTED
 *                otherwise).  The K/V rows are read once per kv head instead of once
 *                per query head.
 * The grouped-head and forced-row rules are readings of the article's §2.3 and
 * §5.2 (which state the scoring and the budget per head) and of its §3.2 and §6
 * tuning advice (some tokens keep full attention); the paged layout follows the
 * block-table caches that paged-attention serving uses.  Same errors and
 * asynchrony as adamas_decode_step; the workspace size is adamas_workspace_bytes of
 * (B, Hq, Hkv, Nmax, d, budget) with Nmax = max_pages * page_size when paged.
 */
typedef struct adamas_decode_args {
    const void *q;
    uint8_t *codes;
    void *K;
    void *V;
    const int32_t *seq_lens;
    int B, Hq, Hkv;
    int64_t Nmax;
    int d;
    int budget;
    float *out;
    int32_t *idx;
    void *workspace;
    size_t workspace_bytes;
    const int32_t *append_pos;
    const void *k_new;
    const void *v_new;
    const int32_t *block_table;
    int64_t n_pages;
    int page_size;
    int max_pages;
    int n_sink;
    int n_recent;
    int policy;
} adamas_decode_args;

int adamas_decode_step_ex(const adamas_decode_args *args, adamas_stream_t stream);

/*
 * Test hook (not for production use): from now on every decode step runs its
 * general kernel and never issues the bulk copy of code stage `stage` in any
 * block, so the workers' bounded wait for that stage gives up after about a
 * second, sets ADAMAS_DEVERR_TIMEOUT and the step completes with invalid outputs;
 * no copy is left in flight.  A negative `stage` turns the hook off.  Process-wide
 * and not thread-safe: for the tests of the timeout path only.
 */
void adamas_debug_withhold_stage(int stage);

/*
 * Sequence-sharded decode step, for contexts longer than one GPU holds (the 2M-token
 * context blog, intelliparadigm.com/.../2174157, §5.1: two million tokens need
 * several GPUs or CPU offloading; the AMD Zebra-HyLo article,
 * yeyulingfeng.com/a/1106654.html, reports 2M-token contexts).  Each of `world`
 * GPUs holds one contiguous slice of every sequence (rank r the r-th slice, in
 * sequence order) in its own codes/K/V arrays, [B][Hkv][Nmax][...] as above with
 * seq_lens[b] the slice's length.  One step, on every rank:
 *   1. adamas_shard_score: scores the slice; writes the slice's distance
 *      histograms to `hist` [B][Hq][ADAMAS_HIST_STRIDE] uint32 (bins 0..384).
 *   2. all-gather of `hist` in rank order -> hist_all [world][B][Hq][ADAMAS_HIST_STRIDE].
 *   3. adamas_shard_attend: from hist_all, the threshold and rank bases of the
 *      whole sequence (k_eff = min(budget, total length)); the slice's kept tokens
 *      get their slots, idx [B][Hq][budget] holds their indices in the whole
 *      sequence (every other slot -1), and `partial` [B][Hq][ADAMAS_PARTIAL_FLOATS]
 *      fp32 receives the slice's softmax state over them.
 *   4. all-gather of `partial` -> [world][B][Hq][ADAMAS_PARTIAL_FLOATS], and an
 *      all-reduce (max) of idx.
 *   5. adamas_merge_partials -> out [B][Hq][128].
 * The result is the step of adamas_decode_step on the whole sequence: the same
 * idx, and out within the float tolerance of the single-GPU step.  Per head and
 * rank the messages are 388 * 4 B (histograms) and 132 * 4 B (state) plus the idx
 * row.  Per-head selection only (no forced rows, paged cache, group-shared policy
 * or append); global indices are int32, so a sequence holds at most 2^31 - 1 tokens.
 *
 * The workspace (adamas_shard_workspace_bytes, initialised once with
 * adamas_workspace_init) carries the slice's distances and per-block histograms
 * from step 1 to step 3: use the same workspace, stream and shape for both.
 * `hist` and idx are overwritten (zeroed / set to -1) by the calls themselves.
 * A partial state is (m, l, 0, 0, o[128]): m the largest score of the slice's kept
 * tokens, in log2 units (q.k / sqrt(128) * log2 e), l = sum 2^(s - m) and
 * o = sum 2^(s - m) v over them; m = -inf and l = 0 when the slice kept none.
 * Errors as for adamas_decode_step; the device error word is the workspace's.
 */
#define ADAMAS_HIST_STRIDE 388
#define ADAMAS_PARTIAL_FLOATS 132

size_t adamas_shard_workspace_bytes(int B, int Hq, int Hkv, int64_t Nmax, int d, int budget);

int adamas_shard_score(const void *q, const uint8_t *codes, const int32_t *seq_lens, int B, int Hq, int Hkv,
                       int64_t Nmax, int d, int budget, uint32_t *hist, void *workspace, size_t workspace_bytes,
                       adamas_stream_t stream);

/* world >= 1 ranks, 0 <= rank < world; hist_all as gathered in step 2. */
int adamas_shard_attend(const void *q, const void *K, const void *V, const int32_t *seq_lens, int B, int Hq, int Hkv,
                        int64_t Nmax, int d, int budget, const uint32_t *hist_all, int world, int rank,
                        float *partial, int32_t *idx, void *workspace, size_t workspace_bytes,
                        adamas_stream_t stream);

/*
 * out[b][h][e] = sum_r 2^(m_r - M) o_r[e] / sum_r 2^(m_r - M) l_r over the n states
 * partials [n][B][Hq][ADAMAS_PARTIAL_FLOATS] (M = max_r m_r; states with m_r = -inf
 * are skipped; 0 when every state is empty).  16-byte aligned fp32 arrays.
 */
int adamas_merge_partials(const float *partials, int n, int B, int Hq, float *out, adamas_stream_t stream);

/*
 * Synchronise `stream`, then copy the workspace's device error word into
 * *error_word (ADAMAS_DEVERR_* bits).  Returns ADAMAS_OK when the word is zero,
 * ADAMAS_ERR_DEVICE when it is not.
 */
int adamas_get_device_error(const void *workspace, size_t workspace_bytes, uint32_t *error_word,
                            adamas_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ADAMAS_H */
