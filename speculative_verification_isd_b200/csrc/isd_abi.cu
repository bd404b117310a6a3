// C-ABI entry points of libisd.so (declared in include/isd.h): host-side
// validation, workspace checks and the launch sequence of one ISD step.  No
// entry point allocates, synchronises or reads device data on the host, so a
// whole step can be captured into a CUDA graph.  One exception: the first
// isd_layers call for a new projection shape times cuBLASLt's candidate
// algorithms on its stream (outside stream capture only).
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include "common.cuh"
#include "plan.h"

namespace {
thread_local char g_last_error[256] = "";
thread_local char g_detail[160] = "";
}  // namespace

namespace isd {
// Host-side context for the next CUDA failure report (this thread).
void set_error_detail(const char* msg) { snprintf(g_detail, sizeof(g_detail), "%s", msg); }
// The message isd_last_error() returns (this thread).
void set_last_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

int persistent_grid() {
    static int sms[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kPlanSMs;
    if (!sms[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        sms[dev] = n < 1 ? kPlanSMs : (n > kMaxSMs ? kMaxSMs : n);
    }
    return sms[dev];
}
cudaError_t launch_attention(const Plan& p, const isd_dims* d, const uint16_t* q,
                             const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_pool,
                             uint16_t* v_pool, const int32_t* page_table, const int32_t* kv_len,
                             const int32_t* n_clean, uint16_t* out, void* ws, int32_t* err_flag,
                             cudaStream_t st, int* clear_extra, int* clear_range, int clear_count,
                             bool pdl, bool bidir);
cudaError_t launch_lm_head(const uint16_t* hidden, const uint16_t* W, int Mh, int H, int V,
                           float* logits, float4* stats_part, void* tail_ws, int32_t* err_flag,
                           cudaStream_t st, bool pdl, bool counters_cleared);
cudaError_t launch_lm_stats_merge(const float4* part, int n_parts, int rows, isd_row_stat* out,
                                  cudaStream_t st, bool pdl);
int lm_head_stat_parts(int Mh, int H, int V);
cudaError_t launch_lora(const Plan& p, const isd_dims* d, const uint16_t* hidden,
                        const uint16_t* lora_A, const uint16_t* lora_B, uint16_t* hidden_out,
                        void* ws, cudaStream_t st, bool pdl);
cudaError_t launch_row_stats(const Plan& p, const float* logits, int rows, int V,
                             isd_row_stat* out, void* ws, cudaStream_t st);
cudaError_t launch_prepare_block(const isd_dims* d, int Q, const uint16_t* Eq, const uint16_t* Ek,
                                 const uint16_t* Ev, const int32_t* n_clean, const int32_t* clean_tok,
                                 bool mask_neg, const float* rope, int rope_len,
                                 const int32_t* kv_len, int32_t* page_table,
                                 int32_t* pages_used, int32_t* next_free, uint16_t* q,
                                 uint16_t* k_new, uint16_t* v_new, int32_t* err_flag,
                                 cudaStream_t st, bool pdl);
cudaError_t gemm_bf16(int M, int Nout, int K, const void* X, const void* W, void* Y, bool acc,
                      void* lt_ws, size_t lt_ws_bytes, void* scratch, size_t scratch_bytes,
                      cudaStream_t st);
cudaError_t launch_rmsnorm(const void* x, const void* w, void* y, int M, int H, float eps,
                           cudaStream_t st);
cudaError_t launch_qk_norm_rope(const isd_dims* d, int Q, const void* qkv, const void* q_norm,
                                const void* k_norm, const float* rope, int rope_len,
                                const int32_t* kv_len, const int32_t* n_clean, float eps, void* q,
                                void* k, void* v, int32_t* err_flag, cudaStream_t st);
cudaError_t launch_silu_mul(const void* gu, void* act, int M, int I, cudaStream_t st);
cudaError_t launch_embed_block(const isd_dims* d, int Q, const void* E, const int32_t* n_clean,
                               const int32_t* clean_tok, void* x, int32_t* err_flag,
                               cudaStream_t st);
cudaError_t launch_sdar_unmask(const isd_dims* d, float tau, bool sync, const float4* stats_part,
                               int n_parts, const isd_row_stat* stats_in, isd_row_stat* stats_out,
                               int32_t* block_tok, int32_t* steps, int32_t* kv_len,
                               int32_t* unmasked, int32_t* out_tok, int32_t* block_steps,
                               int* counters, int32_t* err_flag, cudaStream_t st, bool pdl);
cudaError_t launch_accept(const Plan& p, const isd_dims* d, const float* logits,
                          const isd_row_stat* stats, const float* prev_logits,
                          const isd_row_stat* prev_stats, const int32_t* n_clean,
                          const int32_t* clean_tok, const int32_t* kv_len, const float* uniforms,
                          int32_t* accept_len, int32_t* out_tok, int32_t* next_n_clean,
                          int32_t* next_clean_tok, int32_t* next_kv_len, float* ratio, void* ws,
                          int32_t* err_flag, cudaStream_t st, bool pdl, const float4* stats_part,
                          int n_parts, isd_row_stat* stats_out);
}  // namespace isd

using isd::Plan;

namespace {

isd_status cuda_fail(cudaError_t e) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s%s%s", cudaGetErrorName(e),
             cudaGetErrorString(e), g_detail[0] ? " -- " : "", g_detail);
    g_detail[0] = 0;
    return ISD_ERR_CUDA;
}

isd_status check_ws(const Plan& p, void* ws, size_t ws_bytes) {
    if (!ws || ws_bytes < p.total || (reinterpret_cast<uintptr_t>(ws) & 255)) {
        snprintf(g_last_error, sizeof(g_last_error), "workspace: need %zu bytes, 256-aligned",
                 p.total);
        return ISD_ERR_WORKSPACE;
    }
    return ISD_OK;
}

isd_status invalid(const char* what) {
    snprintf(g_last_error, sizeof(g_last_error), "invalid argument: %s", what);
    return ISD_ERR_INVALID_ARG;
}

isd_status unsupported(const char* what) {
    snprintf(g_last_error, sizeof(g_last_error), "unsupported shape: %s", what);
    return ISD_ERR_UNSUPPORTED_SHAPE;
}

isd_status plan_or_fail(const isd_dims* d, Plan* p) {
    if (!isd::make_plan(d, p)) return invalid("dims");
    return ISD_OK;
}

isd_status check_attention_shape(const isd_dims* d, const Plan& p) {
    if (d->D != 64 && d->D != 128) return unsupported("head dim must be 64 or 128");
    if (p.rows > 128) return unsupported("(Hq/Hkv)*(2N-1) must be <= 128");
    return ISD_OK;
}

isd_status check_lm_shape(const isd_dims* d, const Plan& p, const void* A, const void* Bm) {
    if (p.H % 64) return unsupported("hidden size must be a multiple of 64");
    if (p.M > 512) return unsupported("B*(2N-1) must be <= 512");
    if (d->lora_rank) {
        if (!A || !Bm) return invalid("lora_A/lora_B required when lora_rank > 0");
        if (d->lora_rank % 32 || d->lora_rank > 256)
            return unsupported("lora rank must be a multiple of 32, <= 256");
    } else if (A || Bm) {
        return invalid("lora_A/lora_B given with lora_rank == 0");
    }
    return ISD_OK;
}

isd_status check_accept_shape(const isd_dims* d) {
    if (d->N > 16) return unsupported("stride N must be <= 16");
    static_assert(isd::kAcceptThreads * isd::kAcceptChunk == 524288, "update the message below");
    if ((long long)d->V > (long long)isd::kAcceptThreads * isd::kAcceptChunk)
        return unsupported("vocabulary must be <= 524288 entries");
    return ISD_OK;
}

#define ISD_TRY(x)                        \
    do {                                  \
        isd_status s_ = (x);              \
        if (s_ != ISD_OK) return s_;      \
    } while (0)
#define ISD_CUDA(x)                         \
    do {                                    \
        cudaError_t e_ = (x);               \
        if (e_ != cudaSuccess) return cuda_fail(e_); \
    } while (0)

// The step's kernels are launched with programmatic dependent launch
// (launch.h): each kernel may start its set-up (barriers, TMEM, tensor-map
// prefetch; the LM head also streams W, which no kernel writes) while its
// predecessor finishes, and waits for it before touching anything an earlier
// kernel produces.  At B=32, N=4 on B200 this measured 3 us per step faster
// than plain stream order (paired runs in one process).
constexpr bool kStepPdl = true;

isd_status do_attention(const isd_dims* d, const Plan& p, const uint16_t* q,
                        const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_pool,
                        uint16_t* v_pool, const int32_t* page_table, const int32_t* kv_len,
                        const int32_t* n_clean, uint16_t* out, void* ws, int32_t* err_flag,
                        cudaStream_t st, bool in_step = false, bool bidir = false,
                        bool pdl = false) {
    // n_clean may be null only for a block-causal (SDAR) block, whose N slots are all active
    if (!q || !k_new || !v_new || !k_pool || !v_pool || !page_table || !kv_len ||
        (!n_clean && !bidir) || !out)
        return invalid("null attention pointer");
    ISD_TRY(check_attention_shape(d, p));
    // The launch clears the attention counters on the stream; inside the whole
    // step it also clears the step's accept and LM-head counters.
    int* acc_ticket = nullptr;
    int* lm_ticket = nullptr;
    if (in_step) {
        acc_ticket = reinterpret_cast<int*>(static_cast<char*>(ws) + p.off_acc_ticket);
        lm_ticket = reinterpret_cast<int*>(static_cast<char*>(ws) + p.off_lm_tail +
                                           (size_t)isd::kMaxSMs * isd::lm_part_floats(p.M) * 4);
    }
    ISD_CUDA(isd::launch_attention(p, d, q, k_new, v_new, k_pool, v_pool, page_table, kv_len,
                                   n_clean, out, ws, err_flag, st, acc_ticket, lm_ticket,
                                   in_step ? isd::kMaxSMs : 0, (in_step || pdl) && kStepPdl,
                                   bidir));
    return ISD_OK;
}

isd_status do_lm_head(const isd_dims* d, const Plan& p, const uint16_t* hidden, const uint16_t* W,
                      const uint16_t* lora_A, const uint16_t* lora_B, float* logits,
                      isd_row_stat* row_stats, void* ws, int32_t* err_flag, cudaStream_t st,
                      bool in_step = false) {
    if (!hidden || !W || !logits) return invalid("null lm-head pointer");
    ISD_TRY(check_lm_shape(d, p, lora_A, lora_B));
    const uint16_t* h = hidden;
    if (d->lora_rank) {
        uint16_t* hl = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + p.off_hidden_lora);
        // plain stream order: launched as dependents of the attention, the adapter's
        // kernels measured 7.8 us slower per step at B=64, N=4
        ISD_CUDA(isd::launch_lora(p, d, hidden, lora_A, lora_B, hl, ws, st, false));
        h = hl;
    }
    // Row statistics come out of the LM head's epilogue as partials (one per
    // row and CTA; no second pass over the logits).  On its own the LM head
    // merges them with a small kernel; inside the whole step the accept
    // kernel merges them as it reads them.
    float4* part = row_stats ? reinterpret_cast<float4*>(static_cast<char*>(ws) + p.off_lm_stats)
                             : nullptr;
    ISD_CUDA(isd::launch_lm_head(h, W, p.M, p.H, d->V, logits, part,
                                 static_cast<char*>(ws) + p.off_lm_tail, err_flag, st,
                                 in_step && kStepPdl, in_step));
    if (row_stats && !in_step)
        ISD_CUDA(isd::launch_lm_stats_merge(part, isd::lm_head_stat_parts(p.M, p.H, d->V), p.M,
                                            row_stats, st, false));
    return ISD_OK;
}

}  // namespace

extern "C" {

size_t isd_workspace_bytes(const isd_dims* d) {
    Plan p;
    if (!isd::make_plan(d, &p)) return 0;
    return p.total;
}

const char* isd_status_string(isd_status s) {
    switch (s) {
        case ISD_OK: return "ISD_OK";
        case ISD_ERR_INVALID_ARG: return "ISD_ERR_INVALID_ARG";
        case ISD_ERR_UNSUPPORTED_SHAPE: return "ISD_ERR_UNSUPPORTED_SHAPE";
        case ISD_ERR_WORKSPACE: return "ISD_ERR_WORKSPACE";
        case ISD_ERR_CUDA: return "ISD_ERR_CUDA";
        default: return "ISD_ERR_UNKNOWN";
    }
}

const char* isd_last_error(void) { return g_last_error; }

isd_status isd_attention(const isd_dims* d, const uint16_t* q, const uint16_t* k_new,
                         const uint16_t* v_new, uint16_t* k_pool, uint16_t* v_pool,
                         const int32_t* page_table, const int32_t* kv_len,
                         const int32_t* n_clean, uint16_t* out, void* ws, size_t ws_bytes,
                         int32_t* err_flag, void* stream) {
    Plan p;
    ISD_TRY(plan_or_fail(d, &p));
    ISD_TRY(check_ws(p, ws, ws_bytes));
    return do_attention(d, p, q, k_new, v_new, k_pool, v_pool, page_table, kv_len, n_clean, out,
                        ws, err_flag, static_cast<cudaStream_t>(stream));
}

isd_status isd_lm_head(const isd_dims* d, const uint16_t* hidden, const uint16_t* W,
                       const uint16_t* lora_A, const uint16_t* lora_B, float* logits,
                       isd_row_stat* row_stats, void* ws, size_t ws_bytes, int32_t* err_flag,
                       void* stream) {
    Plan p;
    ISD_TRY(plan_or_fail(d, &p));
    ISD_TRY(check_ws(p, ws, ws_bytes));
    return do_lm_head(d, p, hidden, W, lora_A, lora_B, logits, row_stats, ws, err_flag,
                      static_cast<cudaStream_t>(stream));
}

isd_status isd_row_stats(const isd_dims* d, const float* logits, int32_t rows,
                         isd_row_stat* row_stats, void* ws, size_t ws_bytes, void* stream) {
    Plan p;
    ISD_TRY(plan_or_fail(d, &p));
    ISD_TRY(check_ws(p, ws, ws_bytes));
    if (!logits || !row_stats) return invalid("null row-stats pointer");
    if (rows < 0 || rows > p.M) return invalid("rows must be in [0, B*(2N-1)]");
    if (rows == 0) return ISD_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ISD_CUDA(cudaMemsetAsync(static_cast<char*>(ws) + p.off_stats_ticket, 0, (size_t)p.M * 4, st));
    ISD_CUDA(isd::launch_row_stats(p, logits, rows, d->V, row_stats, ws, st));
    return ISD_OK;
}

// The accept stage; its counters are cleared first unless the caller has
// cleared them on the stream already (the whole step clears them in its
// first kernel).
static isd_status accept_impl(const isd_dims* d, const float* logits, const isd_row_stat* row_stats,
                              const float* prev_logits, const isd_row_stat* prev_row_stats,
                              const int32_t* n_clean, const int32_t* clean_tok, const int32_t* kv_len,
                              const float* uniforms, int32_t* accept_len, int32_t* out_tok,
                              int32_t* next_n_clean, int32_t* next_clean_tok, int32_t* next_kv_len,
                              float* ratio, void* ws, size_t ws_bytes, int32_t* err_flag, void* stream,
                              bool clear_counters, const float4* stats_part = nullptr,
                              int n_parts = 0, isd_row_stat* stats_out = nullptr) {
    Plan p;
    ISD_TRY(plan_or_fail(d, &p));
    ISD_TRY(check_ws(p, ws, ws_bytes));
    ISD_TRY(check_accept_shape(d));
    if (!logits || !row_stats || !prev_logits || !prev_row_stats || !n_clean || !clean_tok ||
        !kv_len || !uniforms || !accept_len || !out_tok || !next_n_clean || !next_clean_tok ||
        !next_kv_len)
        return invalid("null accept pointer");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (clear_counters)
        ISD_CUDA(cudaMemsetAsync(static_cast<char*>(ws) + p.off_acc_ticket, 0, (size_t)d->B * 2 * 4 + 4, st));  // tickets, states, count
    ISD_CUDA(isd::launch_accept(p, d, logits, row_stats, prev_logits, prev_row_stats, n_clean,
                                clean_tok, kv_len, uniforms, accept_len, out_tok, next_n_clean,
                                next_clean_tok, next_kv_len, ratio, ws, err_flag, st,
                                !clear_counters && kStepPdl, stats_part, n_parts, stats_out));
    return ISD_OK;
}

isd_status isd_accept(const isd_dims* d, const float* logits, const isd_row_stat* row_stats,
                      const float* prev_logits, const isd_row_stat* prev_row_stats,
                      const int32_t* n_clean, const int32_t* clean_tok, const int32_t* kv_len,
                      const float* uniforms, int32_t* accept_len, int32_t* out_tok,
                      int32_t* next_n_clean, int32_t* next_clean_tok, int32_t* next_kv_len,
                      float* ratio, void* ws, size_t ws_bytes, int32_t* err_flag, void* stream) {
    return accept_impl(d, logits, row_stats, prev_logits, prev_row_stats, n_clean, clean_tok, kv_len,
                       uniforms, accept_len, out_tok, next_n_clean, next_clean_tok, next_kv_len,
                       ratio, ws, ws_bytes, err_flag, stream, true);
}

}  // extern "C"

// The whole step on validated dims: attention (its first kernel also clears
// the counters of the later ones, so the step issues no memset), LM head,
// accept (which merges this step's row statistics from the LM head's
// partials and writes them to row_stats).
static isd_status step_impl(const isd_dims* d, const Plan& p, const uint16_t* q,
                            const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_pool,
                            uint16_t* v_pool, const int32_t* page_table, const int32_t* kv_len,
                            const int32_t* n_clean, const int32_t* clean_tok, const uint16_t* W,
                            const uint16_t* lora_A, const uint16_t* lora_B, const float* prev_logits,
                            const isd_row_stat* prev_row_stats, const float* uniforms,
                            uint16_t* hidden, float* logits, isd_row_stat* row_stats,
                            int32_t* accept_len, int32_t* out_tok, int32_t* next_n_clean,
                            int32_t* next_clean_tok, int32_t* next_kv_len, float* ratio, void* ws,
                            size_t ws_bytes, int32_t* err_flag, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint16_t* h = hidden ? hidden
                         : reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + p.off_hidden);
    ISD_TRY(do_attention(d, p, q, k_new, v_new, k_pool, v_pool, page_table, kv_len, n_clean, h,
                         ws, err_flag, st, true));
    ISD_TRY(do_lm_head(d, p, h, W, lora_A, lora_B, logits, row_stats, ws, err_flag, st, true));
    const float4* part = reinterpret_cast<const float4*>(static_cast<char*>(ws) + p.off_lm_stats);
    return accept_impl(d, logits, row_stats, prev_logits, prev_row_stats, n_clean, clean_tok,
                       kv_len, uniforms, accept_len, out_tok, next_n_clean, next_clean_tok,
                       next_kv_len, ratio, ws, ws_bytes, err_flag, stream, false, part,
                       isd::lm_head_stat_parts(p.M, p.H, d->V), row_stats);
}

static isd_status check_step(const isd_dims* d, Plan* p, void* ws, size_t ws_bytes,
                             const uint16_t* lora_A, const uint16_t* lora_B) {
    ISD_TRY(plan_or_fail(d, p));
    ISD_TRY(check_ws(*p, ws, ws_bytes));
    ISD_TRY(check_attention_shape(d, *p));
    ISD_TRY(check_lm_shape(d, *p, lora_A, lora_B));
    ISD_TRY(check_accept_shape(d));
    return ISD_OK;
}

extern "C" {

isd_status isd_step(const isd_dims* d, const uint16_t* q, const uint16_t* k_new,
                    const uint16_t* v_new, uint16_t* k_pool, uint16_t* v_pool,
                    const int32_t* page_table, const int32_t* kv_len, const int32_t* n_clean,
                    const int32_t* clean_tok, const uint16_t* W, const uint16_t* lora_A,
                    const uint16_t* lora_B, const float* prev_logits,
                    const isd_row_stat* prev_row_stats, const float* uniforms, uint16_t* hidden,
                    float* logits, isd_row_stat* row_stats, int32_t* accept_len,
                    int32_t* out_tok, int32_t* next_n_clean, int32_t* next_clean_tok,
                    int32_t* next_kv_len, float* ratio, void* ws, size_t ws_bytes,
                    int32_t* err_flag, void* stream) {
    Plan p;
    ISD_TRY(check_step(d, &p, ws, ws_bytes, lora_A, lora_B));
    if (!row_stats || !logits) return invalid("null logits/row_stats");
    return step_impl(d, p, q, k_new, v_new, k_pool, v_pool, page_table, kv_len, n_clean,
                     clean_tok, W, lora_A, lora_B, prev_logits, prev_row_stats, uniforms, hidden,
                     logits, row_stats, accept_len, out_tok, next_n_clean, next_clean_tok,
                     next_kv_len, ratio, ws, ws_bytes, err_flag, stream);
}

static isd_status check_prepare(const isd_dims* d, const uint16_t* Eq, const uint16_t* Ek,
                                const uint16_t* Ev, const void* n_clean, const void* clean_tok,
                                const void* kv_len, const void* page_table, const void* pages_used,
                                const void* next_free, const void* q, const void* k_new,
                                const void* v_new) {
    if (!Eq || !Ek || !Ev || !n_clean || !clean_tok || !kv_len || !page_table || !pages_used ||
        !next_free || !q || !k_new || !v_new)
        return invalid("null prepare-block pointer");
    if ((d->Hkv * d->D) % 8) return unsupported("Hkv * D must be a multiple of 8");
    return ISD_OK;
}

isd_status isd_prepare_block(const isd_dims* d, const uint16_t* Eq, const uint16_t* Ek,
                             const uint16_t* Ev, const int32_t* n_clean, const int32_t* clean_tok,
                             const int32_t* kv_len, int32_t* page_table, int32_t* pages_used,
                             int32_t* next_free_page, uint16_t* q, uint16_t* k_new,
                             uint16_t* v_new, int32_t* err_flag, void* stream) {
    Plan p;
    ISD_TRY(plan_or_fail(d, &p));
    ISD_TRY(check_prepare(d, Eq, Ek, Ev, n_clean, clean_tok, kv_len, page_table, pages_used,
                          next_free_page, q, k_new, v_new));
    ISD_CUDA(isd::launch_prepare_block(d, p.Q, Eq, Ek, Ev, n_clean, clean_tok, false, nullptr, 0,
                                       kv_len,
                                       page_table, pages_used, next_free_page, q, k_new, v_new,
                                       err_flag, static_cast<cudaStream_t>(stream), false));
    return ISD_OK;
}

isd_status isd_loop(const isd_dims* d, int32_t n_steps, const isd_loop_args* a, void* ws,
                    size_t ws_bytes, int32_t* err_flag, void* stream) {
    Plan p;
    if (!a) return invalid("null loop arguments");
    ISD_TRY(check_step(d, &p, ws, ws_bytes, a->lora_A, a->lora_B));
    if (n_steps < 0) return invalid("n_steps must be >= 0");
    ISD_TRY(check_prepare(d, a->Eq, a->Ek, a->Ev, a->n_clean, a->clean_tok, a->kv_len,
                          a->page_table, a->pages_used, a->next_free_page, a->q, a->k_new,
                          a->v_new));
    if (!a->W || !a->k_pool || !a->v_pool || !a->logits || !a->row_stats || !a->uniforms ||
        !a->accept_len_hist || !a->out_tok_hist)
        return invalid("null loop pointer");
    const int B = d->B, N = d->N;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int s = 0; s < n_steps; ++s) {
        const int cur = s & 1, nxt = cur ^ 1;
        ISD_CUDA(isd::launch_prepare_block(
            d, p.Q, a->Eq, a->Ek, a->Ev, a->n_clean + (size_t)cur * B,
            a->clean_tok + (size_t)cur * B * N, false, nullptr, 0, a->kv_len + (size_t)cur * B,
            a->page_table,
            a->pages_used, a->next_free_page, a->q, a->k_new, a->v_new, err_flag, st, kStepPdl));
        ISD_TRY(step_impl(
            d, p, a->q, a->k_new, a->v_new, a->k_pool, a->v_pool, a->page_table,
            a->kv_len + (size_t)cur * B, a->n_clean + (size_t)cur * B,
            a->clean_tok + (size_t)cur * B * N, a->W, a->lora_A, a->lora_B,
            a->logits + (size_t)nxt * p.M * d->V, a->row_stats + (size_t)nxt * p.M,
            a->uniforms + (size_t)s * B * 2 * N, a->hidden, a->logits + (size_t)cur * p.M * d->V,
            a->row_stats + (size_t)cur * p.M, a->accept_len_hist + (size_t)s * B,
            a->out_tok_hist + (size_t)s * B * N, a->n_clean + (size_t)nxt * B,
            a->clean_tok + (size_t)nxt * B * N, a->kv_len + (size_t)nxt * B, nullptr, ws, ws_bytes,
            err_flag, stream));
    }
    return ISD_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// SDAR-style confidence-threshold block decoding (the batch-synchronous
// comparison workload): a block of N query rows with a block-causal mask, the
// same LM head, and the unmask decision kernel (sdar.cu).
// ---------------------------------------------------------------------------
static isd_status check_sdar(const isd_dims* d, Plan* p, void* ws, size_t ws_bytes, float tau) {
    if (!isd::make_plan(d, p, d ? d->N : 0)) return invalid("dims");
    ISD_TRY(check_ws(*p, ws, ws_bytes));
    if (d->N > isd::kSdarMaxN) return unsupported("SDAR block size N must be <= 16");
    if (d->lora_rank) return unsupported("the SDAR workload has no LoRA adapter (lora_rank must be 0)");
    if (!(tau == tau)) return invalid("tau is NaN");
    return ISD_OK;
}

static isd_status sdar_step_impl(const isd_dims* d, const Plan& p, float tau, int32_t sync,
                                 const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                                 uint16_t* k_pool, uint16_t* v_pool, const int32_t* page_table,
                                 int32_t* kv_len, const uint16_t* W, uint16_t* hidden,
                                 float* logits, isd_row_stat* row_stats, int32_t* block_tok,
                                 int32_t* steps, int32_t* unmasked, int32_t* out_tok,
                                 int32_t* block_steps, void* ws, int32_t* err_flag,
                                 cudaStream_t st) {
    if (!W || !logits || !block_tok || !steps || !unmasked || !out_tok || !block_steps)
        return invalid("null SDAR step pointer");
    ISD_TRY(check_attention_shape(d, p));
    ISD_TRY(check_lm_shape(d, p, nullptr, nullptr));
    uint16_t* h = hidden ? hidden
                         : reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + p.off_hidden);
    // KV append + block-causal attention; the append also clears the LM
    // head's counters and the unmask kernel's two counters
    ISD_TRY(do_attention(d, p, q, k_new, v_new, k_pool, v_pool, page_table, kv_len, nullptr, h,
                         ws, err_flag, st, true, true));
    float4* part = reinterpret_cast<float4*>(static_cast<char*>(ws) + p.off_lm_stats);
    ISD_CUDA(isd::launch_lm_head(h, W, p.M, p.H, d->V, logits, part,
                                 static_cast<char*>(ws) + p.off_lm_tail, err_flag, st, kStepPdl,
                                 true));
    int* counters = reinterpret_cast<int*>(static_cast<char*>(ws) + p.off_acc_ticket);
    ISD_CUDA(isd::launch_sdar_unmask(d, tau, sync != 0, part, isd::lm_head_stat_parts(p.M, p.H, d->V),
                                     nullptr, row_stats, block_tok, steps, kv_len, unmasked,
                                     out_tok, block_steps, counters, err_flag, st, kStepPdl));
    return ISD_OK;
}

extern "C" {

isd_status isd_sdar_step(const isd_dims* d, float tau, int32_t sync, const uint16_t* q,
                         const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_pool,
                         uint16_t* v_pool, const int32_t* page_table, int32_t* kv_len,
                         const uint16_t* W, uint16_t* hidden, float* logits,
                         isd_row_stat* row_stats, int32_t* block_tok, int32_t* steps,
                         int32_t* unmasked, int32_t* out_tok, int32_t* block_steps, void* ws,
                         size_t ws_bytes, int32_t* err_flag, void* stream) {
    Plan p;
    ISD_TRY(check_sdar(d, &p, ws, ws_bytes, tau));
    return sdar_step_impl(d, p, tau, sync, q, k_new, v_new, k_pool, v_pool, page_table, kv_len, W,
                          hidden, logits, row_stats, block_tok, steps, unmasked, out_tok,
                          block_steps, ws, err_flag, static_cast<cudaStream_t>(stream));
}

isd_status isd_sdar_unmask(const isd_dims* d, float tau, int32_t sync,
                           const isd_row_stat* row_stats, int32_t* block_tok, int32_t* steps,
                           int32_t* kv_len, int32_t* unmasked, int32_t* out_tok,
                           int32_t* block_steps, void* ws, size_t ws_bytes, int32_t* err_flag,
                           void* stream) {
    Plan p;
    ISD_TRY(check_sdar(d, &p, ws, ws_bytes, tau));
    if (!row_stats || !block_tok || !steps || !kv_len || !unmasked || !out_tok || !block_steps)
        return invalid("null SDAR unmask pointer");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* counters = reinterpret_cast<int*>(static_cast<char*>(ws) + p.off_acc_ticket);
    ISD_CUDA(cudaMemsetAsync(counters, 0, (size_t)d->B * 2 * 4 + 4, st));
    ISD_CUDA(isd::launch_sdar_unmask(d, tau, sync != 0, nullptr, 0, row_stats, nullptr, block_tok,
                                     steps, kv_len, unmasked, out_tok, block_steps, counters,
                                     err_flag, st, false));
    return ISD_OK;
}

isd_status isd_sdar_loop(const isd_dims* d, float tau, int32_t sync, int32_t n_steps,
                         const isd_sdar_loop_args* a, void* ws, size_t ws_bytes,
                         int32_t* err_flag, void* stream) {
    Plan p;
    if (!a) return invalid("null SDAR loop arguments");
    ISD_TRY(check_sdar(d, &p, ws, ws_bytes, tau));
    if (n_steps < 0) return invalid("n_steps must be >= 0");
    ISD_TRY(check_prepare(d, a->Eq, a->Ek, a->Ev, a->block_tok, a->block_tok, a->kv_len,
                          a->page_table, a->pages_used, a->next_free_page, a->q, a->k_new,
                          a->v_new));
    if (!a->unmasked_hist || !a->out_tok_hist || !a->block_steps_hist || !a->steps)
        return invalid("null SDAR loop pointer");
    if (a->rope && (a->rope_positions < 1 || d->D % 16))
        return invalid("rope needs rope_positions >= 1 and D % 16 == 0");
    const int B = d->B, N = d->N;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int s = 0; s < n_steps; ++s) {
        ISD_CUDA(isd::launch_prepare_block(d, p.Q, a->Eq, a->Ek, a->Ev, nullptr, a->block_tok, true,
                                           a->rope, a->rope_positions, a->kv_len, a->page_table, a->pages_used,
                                           a->next_free_page, a->q, a->k_new, a->v_new, err_flag,
                                           st, kStepPdl));
        ISD_TRY(sdar_step_impl(d, p, tau, sync, a->q, a->k_new, a->v_new, a->k_pool, a->v_pool,
                               a->page_table, a->kv_len, a->W, a->hidden, a->logits, a->row_stats,
                               a->block_tok, a->steps, a->unmasked_hist + (size_t)s * B,
                               a->out_tok_hist + (size_t)s * B * N,
                               a->block_steps_hist + (size_t)s * B, ws, err_flag, st));
    }
    return ISD_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Full-depth forward (deep.cu): the decoder stack over the ISD block.  Its
// workspace is the step's (for the attention) followed by the stack's
// activations and the cuBLASLt workspace.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kLtWorkspace = 32u << 20;

struct DeepPlan {
    size_t off_qkv, off_q, off_k, off_v, off_attn, off_h, off_gu, off_act, off_lt, total;
};

bool make_deep_plan(const isd_dims* d, const Plan& p, int inter, DeepPlan* dp) {
    if (inter < 8 || inter % 8) return false;
    const size_t M = (size_t)p.M, D = (size_t)d->D;
    size_t off = isd::align_up(p.total, 256);
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = isd::align_up(off + bytes, 256);
        return o;
    };
    dp->off_qkv = take(M * (d->Hq + 2 * d->Hkv) * D * 2);
    dp->off_q = take(M * d->Hq * D * 2);
    dp->off_k = take(M * d->Hkv * D * 2);
    dp->off_v = take(M * d->Hkv * D * 2);
    dp->off_attn = take(M * p.H * 2);
    dp->off_h = take(M * p.H * 2);
    dp->off_gu = take(M * 2 * (size_t)inter * 2);
    dp->off_act = take(M * (size_t)inter * 2);
    dp->off_lt = take(kLtWorkspace);
    dp->total = off;
    return true;
}
}  // namespace

extern "C" {

isd_status isd_embed_block(const isd_dims* d, const uint16_t* E, const int32_t* n_clean,
                           const int32_t* clean_tok, uint16_t* x, int32_t* err_flag,
                           void* stream) {
    Plan p;
    ISD_TRY(plan_or_fail(d, &p));
    if (!E || !n_clean || !clean_tok || !x) return invalid("null embed-block pointer");
    if (p.H % 8) return unsupported("hidden size must be a multiple of 8");
    ISD_CUDA(isd::launch_embed_block(d, p.Q, E, n_clean, clean_tok, x, err_flag,
                                     static_cast<cudaStream_t>(stream)));
    return ISD_OK;
}

size_t isd_layers_workspace_bytes(const isd_dims* d, int32_t inter) {
    Plan p;
    DeepPlan dp;
    if (!isd::make_plan(d, &p) || !make_deep_plan(d, p, inter, &dp)) return 0;
    return dp.total;
}

isd_status isd_layers(const isd_dims* d, int32_t n_layers, int32_t inter, float eps,
                      const isd_layer* layers, const float* rope, int32_t rope_positions,
                      const uint16_t* final_norm, uint16_t* x, uint16_t* out,
                      const int32_t* page_table, const int32_t* kv_len, const int32_t* n_clean,
                      void* ws, size_t ws_bytes, int32_t* err_flag, void* stream) {
    Plan p;
    DeepPlan dp;
    ISD_TRY(plan_or_fail(d, &p));
    if (!make_deep_plan(d, p, inter, &dp)) return invalid("intermediate size must be a multiple of 8");
    if (!ws || ws_bytes < dp.total || (reinterpret_cast<uintptr_t>(ws) & 255)) {
        snprintf(g_last_error, sizeof(g_last_error),
                 "workspace: need %zu bytes (isd_layers_workspace_bytes), 256-aligned", dp.total);
        return ISD_ERR_WORKSPACE;
    }
    if (n_layers < 0) return invalid("n_layers must be >= 0");
    if (!layers && n_layers) return invalid("null layer array");
    if (!x || !rope || !page_table || !kv_len || !n_clean || (final_norm && !out))
        return invalid("null isd_layers pointer");
    if (rope_positions < 1) return invalid("rope_positions must be >= 1");
    if (p.H % 8) return unsupported("hidden size must be a multiple of 8");
    ISD_TRY(check_attention_shape(d, p));
    for (int l = 0; l < n_layers; ++l) {
        const isd_layer& L = layers[l];
        if (!L.in_norm || !L.w_qkv || !L.q_norm || !L.k_norm || !L.w_o || !L.post_norm ||
            !L.w_gate_up || !L.w_down || !L.k_pool || !L.v_pool)
            return invalid("null pointer in a layer");
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* w = static_cast<char*>(ws);
    void* qkv = w + dp.off_qkv;
    uint16_t* q = reinterpret_cast<uint16_t*>(w + dp.off_q);
    uint16_t* k = reinterpret_cast<uint16_t*>(w + dp.off_k);
    uint16_t* v = reinterpret_cast<uint16_t*>(w + dp.off_v);
    uint16_t* attn = reinterpret_cast<uint16_t*>(w + dp.off_attn);
    void* h = w + dp.off_h;
    void* gu = w + dp.off_gu;
    void* act = w + dp.off_act;
    void* lt = w + dp.off_lt;
    const int M = p.M, H = p.H, qkv_cols = (d->Hq + 2 * d->Hkv) * d->D;
    // the gate/up buffer is free whenever a projection is first tuned (the
    // gate/up projection itself writes it anyway)
    const size_t gu_bytes = (size_t)M * 2 * inter * 2;
    auto gemm = [&](int Nout, int K, const void* X, const void* Wt, void* Y, bool acc) {
        return isd::gemm_bf16(M, Nout, K, X, Wt, Y, acc, lt, kLtWorkspace, gu, gu_bytes, st);
    };
    for (int l = 0; l < n_layers; ++l) {
        const isd_layer& L = layers[l];
        ISD_CUDA(isd::launch_rmsnorm(x, L.in_norm, h, M, H, eps, st));
        ISD_CUDA(gemm(qkv_cols, H, h, L.w_qkv, qkv, false));
        ISD_CUDA(isd::launch_qk_norm_rope(d, p.Q, qkv, L.q_norm, L.k_norm, rope, rope_positions,
                                          kv_len, n_clean, eps, q, k, v, err_flag, st));
        // programmatic dependent launch: the attention's set-up overlaps the K/V append
        ISD_TRY(do_attention(d, p, q, k, v, L.k_pool, L.v_pool, page_table, kv_len, n_clean, attn,
                             ws, err_flag, st, false, false, true));
        ISD_CUDA(gemm(H, H, attn, L.w_o, x, true));
        ISD_CUDA(isd::launch_rmsnorm(x, L.post_norm, h, M, H, eps, st));
        ISD_CUDA(gemm(2 * inter, H, h, L.w_gate_up, gu, false));
        ISD_CUDA(isd::launch_silu_mul(gu, act, M, inter, st));
        ISD_CUDA(gemm(H, inter, act, L.w_down, x, true));
    }
    if (final_norm) ISD_CUDA(isd::launch_rmsnorm(x, final_norm, out, M, H, eps, st));
    return ISD_OK;
}

}  // extern "C"
