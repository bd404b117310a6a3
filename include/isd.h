/*
 * isd.h -- C ABI of the batched ISD (Introspective Strided Decoding)
 * verify-and-propose step for I-DLM, sm_100a (B200).
 *
 * The operation is the one the I-DLM pages describe:
 *   [PRJ] I-DLM project page, Traditional-Chinese text (news.myit.tw/news/ml1xco)
 *   [EXP] "I-DLM：扩散模型如何用“自省一致性”追上自回归模型质量" (blog.hypho.cn)
 *   [ENG] "自省扩散语言模型的 token 生成机制与工程实践" (blog.hotdry.top)
 * One forward over a block of Q = 2N-1 query slots per request verifies the
 * previous stride's N proposals with the p/q criterion min(1, p(x)/q(x)) and
 * proposes the next N tokens ([EXP §Introspective Strided Decoding（ISD）],
 * [ENG §从质量差距到自省机制, §Token 生成的核心参数与验收机制]).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers, owned by the caller, row-major
 *    and densely packed in the layouts stated below.  bf16 tensors are passed
 *    as uint16_t bit patterns.  Nothing is allocated and nothing synchronises:
 *    work is enqueued on `stream` (a cudaStream_t; NULL = legacy default).
 *  - `ws` is caller-owned device scratch of at least isd_workspace_bytes(d)
 *    bytes, 256-byte aligned, with no initial contents required (each call
 *    clears the counters it keeps there on its own stream).  Two calls that
 *    share one workspace must not overlap on the GPU.
 *  - Host-side validation returns a negative isd_status and enqueues nothing.
 *    Data-dependent faults found on the device never trap: they OR a bit into
 *    *err_flag (a device int32 the caller zeroes and reads when it wants) and
 *    the offending request or row is skipped.
 *  - Inputs are never modified, except the KV-pool rows at positions
 *    >= kv_len[b] that the step itself appends; a step can be re-issued on the
 *    same buffers and gives bit-identical results (fixed reduction orders, no
 *    floating-point atomics).
 *
 * Slot layout of the block (Q = 2N-1 rows per request, request-major):
 *   rows 0..N-1 are CLEAN slots: the first c = n_clean[b] hold the tokens
 *   t_1..t_c at positions kv_len..kv_len+c-1, the rest are inactive;
 *   rows N..2N-2 are MASK slots at positions kv_len+c .. kv_len+c+N-2.
 *   By the logit shift ([EXP §三项关键训练创新]) the hidden state of a slot
 *   predicts the token one position later, so t_1 is always accepted
 *   ([PRJ], geometric acceptance paragraph).
 */
#ifndef ISD_H_
#define ISD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t isd_status;
#define ISD_OK                     0
#define ISD_ERR_INVALID_ARG       (-1)  /* null pointer, bad dims or mode */
#define ISD_ERR_UNSUPPORTED_SHAPE (-2)  /* valid but not built: see each call */
#define ISD_ERR_WORKSPACE         (-3)  /* ws too small or misaligned */
#define ISD_ERR_CUDA              (-4)  /* a CUDA launch or driver call failed */

/* Bits OR-ed into *err_flag by the kernels (never a trap). */
#define ISD_FLAG_PAGE_OOB      1  /* a page id outside [0, num_pages) */
#define ISD_FLAG_TOKEN_OOB     2  /* a clean token outside [0, V) */
#define ISD_FLAG_NCLEAN_RANGE  4  /* n_clean outside [1, N] */
#define ISD_FLAG_CAPACITY      8  /* kv_len + block exceeds the request's page capacity */
#define ISD_FLAG_WAIT_TIMEOUT 16  /* a bounded on-chip wait gave up (LM-head pipeline) */

#define ISD_PROPOSE_ARGMAX 0      /* argmax proposals ([ENG §服务部署与 SGLang 集成]) */
#define ISD_PROPOSE_SAMPLE 1      /* inverse-CDF draws with the u_prop uniforms */

typedef struct {
    int32_t B;                  /* requests in the batch */
    int32_t N;                  /* stride; the block has Q = 2N-1 slots */
    int32_t Hq, Hkv, D;         /* query heads, KV heads (Hq % Hkv == 0), head dim */
    int32_t V;                  /* vocabulary size */
    int32_t page_size;          /* tokens per KV page (P) */
    int32_t num_pages;          /* pages in each of k_pool / v_pool */
    int32_t max_pages_per_req;  /* columns of page_table */
    int32_t lora_rank;          /* 0 = no R-ISD adapter, else the rank r */
    int32_t proposal_mode;      /* ISD_PROPOSE_ARGMAX or ISD_PROPOSE_SAMPLE */
    float sm_scale;             /* attention logit scale, usually 1/sqrt(D) */
} isd_dims;

/* Per logits row: max, sum_i exp(z_i - max), argmax (ties -> lowest index). */
typedef struct {
    float max;
    float sumexp;
    int32_t argmax;
    int32_t reserved;
} isd_row_stat;

/* Bytes of scratch needed by any entry point for these dims (isd_step's
 * need is the largest).  Returns 0 for invalid dims. */
size_t isd_workspace_bytes(const isd_dims* d);

/* Static, human-readable name of a status code. */
const char* isd_status_string(isd_status s);

/* Detail of the last failing call on this host thread ("" if none). */
const char* isd_last_error(void);

/*
 * isd_attention -- KV append + strict-causal GQA attention over the paged
 * cache plus the block ([EXP §三项关键训练创新, 严格因果掩码]; paged KV cache
 * per [EXP §推理：复用 AR 推理栈]).
 *   q      [B, Q, Hq, D]  bf16   query vectors of the block slots
 *   k_new  [B, Q, Hkv, D] bf16   keys of the block slots
 *   v_new  [B, Q, Hkv, D] bf16   values of the block slots
 *   k_pool, v_pool [num_pages, page_size, Hkv, D] bf16, in/out: the active
 *          slots' K/V rows are written at their positions (page
 *          page_table[b][pos / P], row pos % P)
 *   page_table [B, max_pages_per_req] int32; kv_len [B] int32 (cached
 *          prefix length); n_clean [B] int32 (c in [1, N])
 *   out    [B*Q, Hq*D] bf16: for each active slot s and head h, the softmax
 *          (sm_scale q.k) weighted sum of v over keys at positions <= pos_s,
 *          query head h reading KV head h / (Hq/Hkv); inactive slots -> 0.
 * Supported: D in {64, 128}; (Hq/Hkv)*Q <= 128.  D = 128 with (Hq/Hkv)*Q
 * <= 64 and page sizes 8, 16, 32, 64 or 128 run on the tensor cores
 * (tcgen05); other supported shapes on a general (mma.sync) kernel.  Both
 * give results that do not depend on timing (fixed-order merges).
 */
isd_status isd_attention(const isd_dims* d, const uint16_t* q, const uint16_t* k_new,
                         const uint16_t* v_new, uint16_t* k_pool, uint16_t* v_pool,
                         const int32_t* page_table, const int32_t* kv_len,
                         const int32_t* n_clean, uint16_t* out, void* ws, size_t ws_bytes,
                         int32_t* err_flag, void* stream);

/*
 * isd_lm_head -- (optional R-ISD gated LoRA on MASK rows) + LM head + row
 * statistics.  [EXP §ISD 核心逻辑伪代码] maps every slot to a vocabulary
 * distribution; [ENG §Token 生成的核心参数与验收机制] and [PRJ] (R-ISD) apply
 * the rank-r gated adapter at MASK positions only.
 *   hidden [B*Q, H] bf16 (H = Hq*D)
 *   W      [V, H] bf16
 *   lora_A [H, r] bf16, lora_B [r, H] bf16 (both NULL iff lora_rank == 0):
 *          MASK rows use h' = bf16(h + bf16(h A) B); clean rows use h.
 *   logits [B*Q, V] fp32 = h' . W^T (fp32 accumulation on tensor cores)
 *   row_stats [B*Q] isd_row_stat, or NULL to skip the statistics.
 * Supported: H % 64 == 0, B*Q <= 512, V >= 1.
 */
isd_status isd_lm_head(const isd_dims* d, const uint16_t* hidden, const uint16_t* W,
                       const uint16_t* lora_A, const uint16_t* lora_B, float* logits,
                       isd_row_stat* row_stats, void* ws, size_t ws_bytes, int32_t* err_flag,
                       void* stream);

/* isd_row_stats -- row statistics of `rows` fp32 logits rows of length V. */
isd_status isd_row_stats(const isd_dims* d, const float* logits, int32_t rows,
                         isd_row_stat* row_stats, void* ws, size_t ws_bytes, void* stream);

/*
 * isd_accept -- p/q verification, residual draw, next-stride proposals and
 * state update ([EXP §Introspective Strided Decoding（ISD）];
 * [ENG §从质量差距到自省机制]).  For request b with c = n_clean[b]:
 *   for j = 2..c: x = t_j, p = softmax(logits row (b, j-2)), q = softmax
 *   (prev_logits row (b, N+j-2)); accept iff u_acc[j-2] < p(x)/q(x); the
 *   first rejection stops.  On a rejection at j the replacement is drawn by
 *   inverse CDF from max(0, p - q) with u_res (argmax p if that mass is 0);
 *   otherwise the next proposals are x'_1 from row (b, c-1) and x'_{m+2} from
 *   row (b, N+m) (argmax, or inverse CDF with u_prop in sample mode).
 *   logits, prev_logits [B, Q, V] fp32 (this and the previous step's)
 *   row_stats, prev_row_stats [B*Q] isd_row_stat of those logits
 *   n_clean [B], clean_tok [B, N], kv_len [B] int32
 *   uniforms [B, 2N] fp32 in [0,1): u_acc[0..N-2], u_res[N-1], u_prop[N..2N-1]
 * Outputs (int32):
 *   accept_len [B] = A = 1 + accepted proposals = tokens emitted this step
 *   out_tok [B, N]: t_2..t_A then the replacement (or x'_1); -1 padded
 *   next_n_clean [B] (1 after a rejection, else N); next_clean_tok [B, N]
 *   (-1 padded); next_kv_len [B] = kv_len + A
 *   ratio [B, max(N-1,1)] fp32 or NULL: p/q of each tested proposal, -1 if
 *   not tested.
 * Supported: N <= 16, V <= 524288 (else ISD_ERR_UNSUPPORTED_SHAPE).
 */
isd_status isd_accept(const isd_dims* d, const float* logits, const isd_row_stat* row_stats,
                      const float* prev_logits, const isd_row_stat* prev_row_stats,
                      const int32_t* n_clean, const int32_t* clean_tok, const int32_t* kv_len,
                      const float* uniforms, int32_t* accept_len, int32_t* out_tok,
                      int32_t* next_n_clean, int32_t* next_clean_tok, int32_t* next_kv_len,
                      float* ratio, void* ws, size_t ws_bytes, int32_t* err_flag, void* stream);

/*
 * isd_step -- the whole step: isd_attention, then isd_lm_head (with row
 * statistics), then isd_accept, enqueued back to back on `stream`.
 * `hidden` [B*Q, H] bf16 receives the attention output if non-NULL (else it
 * stays in ws).  `logits` and `row_stats` are outputs of this step and become
 * the caller's prev_logits / prev_row_stats for the next one.
 * The step issues no memset and no host synchronisation: its first kernel
 * also clears the counters the later kernels use.
 */
isd_status isd_step(const isd_dims* d, const uint16_t* q, const uint16_t* k_new,
                    const uint16_t* v_new, uint16_t* k_pool, uint16_t* v_pool,
                    const int32_t* page_table, const int32_t* kv_len, const int32_t* n_clean,
                    const int32_t* clean_tok, const uint16_t* W, const uint16_t* lora_A,
                    const uint16_t* lora_B, const float* prev_logits,
                    const isd_row_stat* prev_row_stats, const float* uniforms,
                    uint16_t* hidden, float* logits, isd_row_stat* row_stats,
                    int32_t* accept_len, int32_t* out_tok, int32_t* next_n_clean,
                    int32_t* next_clean_tok, int32_t* next_kv_len, float* ratio, void* ws,
                    size_t ws_bytes, int32_t* err_flag, void* stream);

/*
 * isd_prepare_block -- the block activations of one step from each request's
 * state, and on-device page bookkeeping.  The pages give no layer internals,
 * so the per-layer forward that turns the block's tokens into q, k and v is
 * stood in for by a table lookup:
 *   Eq [V+1, Hq, D], Ek, Ev [V+1, Hkv, D] bf16: row t is token t, row V the
 *   MASK token; slot s < n_clean[b] of request b reads row clean_tok[b][s],
 *   every other slot (inactive clean slots, MASK slots) row V.
 *   q [B, Q, Hq, D], k_new, v_new [B, Q, Hkv, D] bf16 (outputs)
 * Page bookkeeping: request b's pages page_table[b][0 .. pages_used[b]) are
 * extended to ceil((kv_len[b] + Q) / P) pages (at most max_pages_per_req)
 * with pages taken in request order from *next_free_page (a bump allocator
 * over [*next_free_page, num_pages), updated).  Running out of pages or
 * columns raises ISD_FLAG_CAPACITY; an out-of-range token ISD_FLAG_TOKEN_OOB
 * (the slot reads the MASK row).
 */
isd_status isd_prepare_block(const isd_dims* d, const uint16_t* Eq, const uint16_t* Ek,
                             const uint16_t* Ev, const int32_t* n_clean, const int32_t* clean_tok,
                             const int32_t* kv_len, int32_t* page_table, int32_t* pages_used,
                             int32_t* next_free_page, uint16_t* q, uint16_t* k_new,
                             uint16_t* v_new, int32_t* err_flag, void* stream);

/*
 * isd_loop -- n_steps ISD steps of a stationary batch, enqueued back to back
 * with no host read between them: each step is isd_prepare_block followed by
 * isd_step on the state of that step, so every request advances on its own
 * ([PRJ], the paragraph on requests advancing independently; [ENG
 * §服务部署与 SGLang 集成]: stationary batch, CUDA-graph capture).  The call is
 * capturable into a CUDA graph.
 * State and outputs are double buffers; step s reads buffer s & 1 and writes
 * buffer (s + 1) & 1 (so the final state is in buffer n_steps & 1):
 *   kv_len [2][B], n_clean [2][B], clean_tok [2][B][N] int32
 *   logits [2][B*Q][V] fp32, row_stats [2][B*Q]: step s writes buffer s & 1
 *          and reads buffer (s + 1) & 1 as the previous step's (step 0 reads
 *          buffer 1, needed only for requests with n_clean > 1)
 *   uniforms [n_steps][B][2N] fp32 (as isd_accept's, per step)
 *   accept_len_hist [n_steps][B], out_tok_hist [n_steps][B][N] int32: the
 *          accept lengths and emitted tokens of every step
 *   q, k_new, v_new, hidden: one block's activations (caller-owned scratch,
 *          the sizes of isd_step's arguments); page_table, pages_used,
 *          next_free_page, k_pool, v_pool, W, lora_A, lora_B, Eq, Ek, Ev as
 *          in isd_prepare_block and isd_step.
 * ws: isd_workspace_bytes(d) bytes, as for isd_step.
 * Ownership: every buffer is the caller's device memory; the call allocates
 * nothing and reads nothing back to the host.
 * Errors: invalid dims, a null pointer among the required ones (lora_A and
 * lora_B may be null when lora_rank is 0), n_steps < 0 or a short workspace
 * return ISD_ERR_* before anything is enqueued; a launch failure part-way
 * returns ISD_ERR_CUDA with the earlier steps enqueued.  Device-side faults
 * (a page or token out of range, a request out of pages) set err_flag bits
 * and never trap; the affected requests carry their state over.
 */
typedef struct {
    const uint16_t* Eq;
    const uint16_t* Ek;
    const uint16_t* Ev;
    const uint16_t* W;
    const uint16_t* lora_A;
    const uint16_t* lora_B;
    uint16_t* k_pool;
    uint16_t* v_pool;
    int32_t* page_table;
    int32_t* pages_used;
    int32_t* next_free_page;
    int32_t* kv_len;
    int32_t* n_clean;
    int32_t* clean_tok;
    float* logits;
    isd_row_stat* row_stats;
    const float* uniforms;
    uint16_t* q;
    uint16_t* k_new;
    uint16_t* v_new;
    uint16_t* hidden;
    int32_t* accept_len_hist;
    int32_t* out_tok_hist;
} isd_loop_args;

isd_status isd_loop(const isd_dims* d, int32_t n_steps, const isd_loop_args* a, void* ws,
                    size_t ws_bytes, int32_t* err_flag, void* stream);

/*
 * isd_attention_noalloc -- isd_attention for callers that cannot provide a
 * workspace.  The pages have no counterpart: this is a deployment convenience.
 *
 * Some callers cannot allocate device memory for us: a serving engine that
 * gave all free device memory to its KV-cache pool at start-up, or code that
 * must not call the CUDA allocator (cudaMalloc/cudaFree can synchronise the
 * device).  This call takes the same inputs and outputs as isd_attention, but
 * its scratch (the attention's partial results and counters) lives in a fixed
 * array inside the library of ISD_NOALLOC_SCRATCH_BYTES bytes, which every
 * GPU that loads the library keeps until the process exits.  It allocates
 * nothing and calls no allocating routine.
 *  - Dims whose scratch need exceeds ISD_NOALLOC_SCRATCH_BYTES are rejected
 *    with ISD_ERR_WORKSPACE (isd_last_error() states both sizes).  The need
 *    grows with B * Hkv * (longest context); B=32, 8 KV heads and 8 K
 *    contexts fit.
 *  - The first call on each device (made with that device current) looks up
 *    the array's device address, and so does the first call after the
 *    device's context was destroyed and recreated (cudaDeviceReset); make
 *    those calls before any stream capture.
 *  - All calls on a device share the array: calls that overlap on the GPU
 *    (e.g. on two unordered streams) race on it.  Each call clears the
 *    counters it needs on its own stream.
 */
#define ISD_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
isd_status isd_attention_noalloc(const isd_dims* d, const uint16_t* q, const uint16_t* k_new,
                                 const uint16_t* v_new, uint16_t* k_pool, uint16_t* v_pool,
                                 const int32_t* page_table, const int32_t* kv_len,
                                 const int32_t* n_clean, uint16_t* out, int32_t* err_flag,
                                 void* stream);

/*
 * ---------------------------------------------------------------------------
 * SDAR-style confidence-threshold block decoding: the batch-synchronous
 * comparison workload.  The I-DLM project page (paragraphs comparing ISD with
 * SDAR) says SDAR denoises a block of N positions by confidence with N queries
 * per forward, and that a batch waits for its slowest block, so a round costs
 * max(S_1..S_B) forwards, a cost ISD does not pay.  The rule is not spelled
 * out; these calls take the plain reading:
 *  - block: positions kv_len .. kv_len+N-1, all N rows computed every forward;
 *    a committed position carries its token, an uncommitted one MASK;
 *  - attention is block-causal: every block row sees the prefix and all N
 *    rows of its block; each forward writes the N rows' K/V at their
 *    positions, and they stay in the cache when the block is committed;
 *  - row s predicts position s; confidence = the row's largest softmax
 *    probability, fl32(1) / fl32(sum_i exp(z_i - max)); candidate = argmax;
 *  - unmask: every uncommitted position with confidence >= tau commits its
 *    candidate; if none does, the most confident uncommitted one does (ties:
 *    lowest position); a block takes S_b in [1, N] such forwards;
 *  - a complete block gets one more forward over its final tokens (its
 *    store pass: the K/V that forward appends stay in the cache), after
 *    which it may leave: kv_len += N, a fresh block of MASK;
 *  - sync != 0: the batch moves on only when every request's block is
 *    complete and stored (a round costs max_b S_b + 1 forwards); requests
 *    that finished early idle.  sync == 0: each stored block moves on by
 *    itself (S_b + 1 forwards).
 * Dims: isd_dims with N = the block size (<= 16) and lora_rank 0; the block
 * has Q = N rows (not 2N-1).  isd_workspace_bytes(d) covers these calls.
 * State (device, int32, updated in place): block_tok [B, N] (-1 = MASK),
 * steps [B] (forwards spent on the current block), kv_len [B].
 * Per call outputs: unmasked [B] (positions committed by this forward),
 * out_tok [B, N] (a block's tokens when it leaves the batch in this call,
 * else -1), block_steps [B] (its S_b, denoising forwards without the store
 * pass, then; else 0).
 * Ownership: every pointer is the caller's device memory (the state buffers
 * are read and written in place); nothing is allocated, nothing is read on
 * the host, and the calls are capturable.
 * Errors: invalid pointers or dims -> ISD_ERR_INVALID_ARG; N > 16, lora_rank
 * != 0 or shapes the attention / LM head do not support ->
 * ISD_ERR_UNSUPPORTED_SHAPE; a workspace too small or misaligned ->
 * ISD_ERR_WORKSPACE.  On the device, a page id outside the pool
 * raises ISD_FLAG_PAGE_OOB, a block that does not fit the request's pages
 * ISD_FLAG_CAPACITY, a committed token outside [0, V) ISD_FLAG_TOKEN_OOB.
 * ---------------------------------------------------------------------------
 */

/*
 * isd_sdar_step -- one forward and decision of the batch: KV append +
 * block-causal attention, LM head (logits [B*N, V] fp32), row statistics
 * (row_stats [B*N], optional), unmask.  q [B, N, Hq, D], k_new / v_new
 * [B, N, Hkv, D] bf16; pools, page_table as for isd_attention; hidden
 * [B*N, H] bf16 or NULL (workspace).  No host synchronisation; capturable.
 */
isd_status isd_sdar_step(const isd_dims* d, float tau, int32_t sync, const uint16_t* q,
                         const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_pool,
                         uint16_t* v_pool, const int32_t* page_table, int32_t* kv_len,
                         const uint16_t* W, uint16_t* hidden, float* logits,
                         isd_row_stat* row_stats, int32_t* block_tok, int32_t* steps,
                         int32_t* unmasked, int32_t* out_tok, int32_t* block_steps, void* ws,
                         size_t ws_bytes, int32_t* err_flag, void* stream);

/*
 * isd_sdar_unmask -- the decision alone, on given row statistics
 * (row_stats [B*N]); same state and outputs as isd_sdar_step.
 */
isd_status isd_sdar_unmask(const isd_dims* d, float tau, int32_t sync,
                           const isd_row_stat* row_stats, int32_t* block_tok, int32_t* steps,
                           int32_t* kv_len, int32_t* unmasked, int32_t* out_tok,
                           int32_t* block_steps, void* ws, size_t ws_bytes, int32_t* err_flag,
                           void* stream);

/*
 * isd_sdar_loop -- n_steps forwards of a stationary batch on the device, each
 * one: block activations by table lookup (Eq/Ek/Ev [V+1, heads, D], row V =
 * MASK, as isd_prepare_block does for an ISD block) with the page list grown
 * to cover kv_len + N, then isd_sdar_step on the state in place.  Step s
 * writes unmasked_hist[s] [B], out_tok_hist[s] [B, N], block_steps_hist[s]
 * [B]; logits, row_stats, q, k_new, v_new and hidden hold the last step's.
 * rope (optional): [rope_positions, D/2, 2] fp32 (cos, sin) per position and
 * pair; when given, the q and k rows of block position s are rotated by
 * position kv_len + s (pairs (i, i + D/2), each product and sum rounded in
 * fp32, then to bf16), as a rotary-embedded model's are; a position past the
 * table raises ISD_FLAG_CAPACITY and is left unrotated.  NULL: no rotation.
 * Ownership: every pointer is the caller's device memory, which must stay
 * valid until the enqueued work completes; nothing is allocated.
 */
typedef struct {
    const uint16_t* Eq;
    const uint16_t* Ek;
    const uint16_t* Ev;
    const uint16_t* W;
    uint16_t* k_pool;
    uint16_t* v_pool;
    int32_t* page_table;
    int32_t* pages_used;
    int32_t* next_free_page;
    int32_t* kv_len;
    int32_t* block_tok;
    int32_t* steps;
    float* logits;
    isd_row_stat* row_stats;
    uint16_t* q;
    uint16_t* k_new;
    uint16_t* v_new;
    uint16_t* hidden;
    int32_t* unmasked_hist;
    int32_t* out_tok_hist;
    int32_t* block_steps_hist;
    const float* rope;
    int32_t rope_positions;
} isd_sdar_loop_args;

isd_status isd_sdar_loop(const isd_dims* d, float tau, int32_t sync, int32_t n_steps,
                         const isd_sdar_loop_args* a, void* ws, size_t ws_bytes,
                         int32_t* err_flag, void* stream);

/*
 * ---------------------------------------------------------------------------
 * isd_layers -- the full-depth forward over the ISD block: the decoder stack
 * that the single-layer step stands in for.  I-DLM keeps the AR model's stack
 * and serving path ([EXP §推理：复用 AR 推理栈]; its 8B model is built from
 * Qwen3-8B); the layer internals are not in the pages and follow the base
 * model (Qwen3) decoder layer, over all 2N-1 slots of the block at once:
 *   x += O(attn(RoPE(qk_norm(QKV(rmsnorm_in(x))))))
 *   x += down(silu(gate(h)) * up(h)),  h = rmsnorm_post(x)
 * then, if final_norm is given, out = rmsnorm_final(x) (the LM head's input).
 *  - attention: isd_attention's slot layout, strict-causal mask and paged
 *    K/V append, with each layer's own pools (one page table for all);
 *  - q and k are RMS-normalised per head (q_norm, k_norm over D) and rotated
 *    by the slot's position (clean slot s: kv_len + s; MASK slot m:
 *    kv_len + c + m) with rope [rope_positions, D/2, 2] fp32 (cos, sin),
 *    rotate-half pairs (i, i + D/2); a position past the table raises
 *    ISD_FLAG_CAPACITY (the last row is used);
 *  - RMSNorm: x / sqrt(mean(x^2) + eps) * w, statistics in fp32;
 *  - rounding to bf16 at every norm output, every GEMM output (the O and
 *    down projections add the residual first), q / k after norm + rotation,
 *    the attention output and silu(gate) * up; fp32 in between.  The four
 *    projections run on cuBLASLt (bf16, fp32 accumulation).
 * Shapes: H = Hq * D (multiple of 8), D in {64, 128}; x, out [B*(2N-1), H]
 * bf16 (x is the residual stream, in/out); layers: a HOST array of n_layers
 * isd_layer, each holding device pointers: in_norm, post_norm [H]; w_qkv
 * [(Hq + 2 Hkv) D, H] (q rows, then k, then v); q_norm, k_norm [D]; w_o
 * [H, Hq D]; w_gate_up [2 inter, H] (gate rows first); w_down [H, inter];
 * k_pool, v_pool [num_pages, page_size, Hkv, D].
 * Workspace: isd_layers_workspace_bytes(d, inter) bytes, 256-aligned (the
 * first isd_workspace_bytes(d) of it serve the attention).  The first call
 * for a new projection shape queries cuBLASLt's heuristic and times its
 * best candidates on the call's stream (this synchronises that stream once;
 * the fastest is kept for the process); make it before any stream capture
 * (under capture, the heuristic's first choice is used).
 * Ownership: the layer array is the caller's host memory, read during the
 * call only; every pointer in it and every other pointer is the caller's
 * device memory; nothing is allocated.
 * Errors: invalid dims, a null pointer, n_layers < 0, inter not a multiple
 * of 8 or rope_positions < 1 -> ISD_ERR_INVALID_ARG; H not a multiple of 8
 * or an attention shape isd_attention does not support ->
 * ISD_ERR_UNSUPPORTED_SHAPE; a workspace below isd_layers_workspace_bytes or
 * misaligned -> ISD_ERR_WORKSPACE; a cuBLASLt failure -> ISD_ERR_CUDA
 * (isd_last_error() names it).
 */
typedef struct {
    const uint16_t* in_norm;
    const uint16_t* w_qkv;
    const uint16_t* q_norm;
    const uint16_t* k_norm;
    const uint16_t* w_o;
    const uint16_t* post_norm;
    const uint16_t* w_gate_up;
    const uint16_t* w_down;
    uint16_t* k_pool;
    uint16_t* v_pool;
} isd_layer;

size_t isd_layers_workspace_bytes(const isd_dims* d, int32_t inter);

/*
 * isd_embed_block -- the block's input embeddings for isd_layers: slot s of
 * request b takes row E[t] of the embedding table E [V+1, H] bf16 (row V =
 * MASK) for an active clean slot (s < n_clean[b]; t = clean_tok[b][s]), the
 * MASK row for inactive clean slots and every MASK slot.  x [B*(2N-1), H].
 * A token outside [0, V) raises ISD_FLAG_TOKEN_OOB (the MASK row is used).
 * Ownership: caller's device memory throughout.  Errors: invalid dims or a
 * null pointer -> ISD_ERR_INVALID_ARG; H not a multiple of 8 ->
 * ISD_ERR_UNSUPPORTED_SHAPE.
 */
isd_status isd_embed_block(const isd_dims* d, const uint16_t* E, const int32_t* n_clean,
                           const int32_t* clean_tok, uint16_t* x, int32_t* err_flag,
                           void* stream);

isd_status isd_layers(const isd_dims* d, int32_t n_layers, int32_t inter, float eps,
                      const isd_layer* layers, const float* rope, int32_t rope_positions,
                      const uint16_t* final_norm, uint16_t* x, uint16_t* out,
                      const int32_t* page_table, const int32_t* kv_len, const int32_t* n_clean,
                      void* ws, size_t ws_bytes, int32_t* err_flag, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ISD_H_ */
