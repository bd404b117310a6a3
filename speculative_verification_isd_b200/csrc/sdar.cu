// SDAR-style confidence-threshold block decoding: the decision kernel of the
// batch-synchronous comparison workload of the I-DLM pages.
//
// The I-DLM project page (the paragraphs comparing ISD with SDAR) says that
// SDAR denoises a block of N positions by confidence, one forward of N
// queries per denoising step, and that a batch has to wait for its slowest
// block: the forwards a round costs are max(S_1..S_B), whose mean grows with
// the batch size, while ISD requests advance on their own.  The rule is named,
// not spelled out; this kernel takes the plain reading:
//   - confidence of block position s = the largest softmax probability of
//     its row, 1 / sum_i exp(z_i - max z), candidate = the row's argmax;
//   - every uncommitted position with confidence >= tau commits its
//     candidate; if none does, the single most confident uncommitted one
//     does (ties to the lowest position), so a block takes 1..N denoising
//     forwards;
//   - a complete block gets one more forward over its final tokens (its
//     store pass: the K/V rows that forward appends are the ones the cache
//     keeps), after which it may leave (kv_len += N, block reset to MASK);
//   - with sync, the batch moves to the next block only once every request's
//     block is complete and stored; without it each request moves on by itself.
// One CTA per request, one warp per block row: the warp merges the row's
// statistics from the LM head's partials (the routine and order every other
// merge of the library uses), lane 0 forms the confidence in float32, and
// thread 0 takes the request's decisions.  Under sync the CTA that draws the
// last ticket commits the batch (last-block-done pattern: nothing spins).
#include "common.cuh"
#include "launch.h"
#include "plan.h"

namespace isd {

struct SdarArgs {
    int B, N, V, sync;
    float tau;
    const float4* stats_part;     // [B*N][n_parts] LM-head partials, or null
    int n_parts;
    const isd_row_stat* stats_in; // merged statistics, when stats_part is null
    isd_row_stat* stats_out;      // merged statistics (optional)
    int32_t* block_tok;           // [B, N] in/out, -1 = MASK
    int32_t* steps;               // [B] in/out: forwards spent on the current block
    int32_t* kv_len;              // [B] in/out
    int32_t* unmasked;            // [B] out: positions committed by this forward
    int32_t* out_tok;             // [B, N] out: the block's tokens if it left the batch now, else -1
    int32_t* block_steps;         // [B] out: its S_b then, else 0
    int* ticket;                  // zero on entry; reset by the last CTA
    int* done_count;              // zero on entry; reset by the last CTA
    int32_t* err_flag;
};

__global__ void __launch_bounds__(32 * kSdarMaxN) sdar_unmask_kernel(const __grid_constant__ SdarArgs a) {
    pdl_trigger();
    pdl_wait();  // the LM head's partials
    const int b = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = a.N;
    __shared__ float s_conf[kSdarMaxN];
    __shared__ int s_cand[kSdarMaxN];
    __shared__ int s_last;
    if (warp < N) {
        const int row = b * N + warp;
        RowStat st;
        if (a.stats_part) {
            st = warp_merge_partials<4>(a.stats_part + (size_t)row * a.n_parts, a.n_parts);
        } else {
            const isd_row_stat r = a.stats_in[row];
            st = RowStat{r.max, r.sumexp, r.argmax};
        }
        if (lane == 0) {
            if (a.stats_out) a.stats_out[row] = isd_row_stat{st.m, st.s, st.idx, 0};
            s_conf[warp] = __fdiv_rn(1.f, st.s);
            s_cand[warp] = st.idx;
        }
    }
    __syncthreads();
    int32_t* tok = a.block_tok + (size_t)b * N;
    if (threadIdx.x == 0) {
        // decisions of request b
        int n_commit = 0, best = -1;
        uint32_t open = 0;
        for (int s = 0; s < N; ++s) {
            const int t = tok[s];
            if (t < 0) {
                open |= 1u << s;
            } else if (t >= a.V) {
                raise_flag(a.err_flag, ISD_FLAG_TOKEN_OOB);
            }
        }
        int steps = a.steps[b];
        if (open) {
            for (int s = 0; s < N; ++s) {
                if (!(open >> s & 1)) continue;
                if (s_conf[s] >= a.tau) {
                    tok[s] = s_cand[s];
                    ++n_commit;
                } else if (best < 0 || s_conf[s] > s_conf[best]) {
                    best = s;  // the most confident position that did not clear tau
                }
            }
            if (n_commit == 0) {
                tok[best] = s_cand[best];
                n_commit = 1;
            }
            ++steps;
        }
        // complete when this forward began: this forward was its store pass
        const bool stored = open == 0;
        a.unmasked[b] = n_commit;
        int32_t* out = a.out_tok + (size_t)b * N;
        if (!a.sync && stored) {
            // without sync a stored block leaves the batch at once
            for (int s = 0; s < N; ++s) {
                out[s] = tok[s];
                tok[s] = -1;
            }
            a.block_steps[b] = steps;
            a.steps[b] = 0;
            a.kv_len[b] += N;
        } else {
            for (int s = 0; s < N; ++s) out[s] = -1;
            a.block_steps[b] = 0;
            a.steps[b] = steps;
        }
        if (a.sync) {
            if (stored) atomicAdd(a.done_count, 1);
            __threadfence();
            s_last = atomicAdd(a.ticket, 1) == a.B - 1;
        }
    }
    if (!a.sync) return;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const bool all_done = __ldcg(a.done_count) == a.B;
    __syncthreads();  // every thread has read the count before it is reset
    if (all_done) {
        // the batch's round is over: every block leaves, the next one starts
        for (int i = threadIdx.x; i < a.B * N; i += blockDim.x) {
            const int t = __ldcg(a.block_tok + i);
            a.out_tok[i] = t;
            a.block_tok[i] = -1;
        }
        for (int r = threadIdx.x; r < a.B; r += blockDim.x) {
            a.block_steps[r] = __ldcg(a.steps + r);
            a.steps[r] = 0;
            a.kv_len[r] = __ldcg(a.kv_len + r) + N;
        }
    }
    if (threadIdx.x == 0) {
        *a.ticket = 0;
        *a.done_count = 0;
    }
}

cudaError_t launch_sdar_unmask(const isd_dims* d, float tau, bool sync, const float4* stats_part,
                               int n_parts, const isd_row_stat* stats_in, isd_row_stat* stats_out,
                               int32_t* block_tok, int32_t* steps, int32_t* kv_len,
                               int32_t* unmasked, int32_t* out_tok, int32_t* block_steps,
                               int* counters, int32_t* err_flag, cudaStream_t st, bool pdl) {
    SdarArgs a;
    a.B = d->B;
    a.N = d->N;
    a.V = d->V;
    a.sync = sync ? 1 : 0;
    a.tau = tau;
    a.stats_part = stats_part;
    a.n_parts = n_parts;
    a.stats_in = stats_in;
    a.stats_out = stats_out;
    a.block_tok = block_tok;
    a.steps = steps;
    a.kv_len = kv_len;
    a.unmasked = unmasked;
    a.out_tok = out_tok;
    a.block_steps = block_steps;
    // the two counters sit where the step's first kernel clears them: the
    // first of the B accept tickets and the decided count after 2B ints
    a.ticket = counters;
    a.done_count = counters + 2 * d->B;
    a.err_flag = err_flag;
    return launch_kernel(pdl, sdar_unmask_kernel, dim3(d->B), dim3(32 * d->N), 0, st, a);
}

}  // namespace isd
