// Row statistics (a5) and the fused p/q accept / residual draw / proposal /
// state-update kernel (a6-a9) of the ISD step.
//
// Verification follows the p/q criterion min(1, p(x)/q(x)) of the I-DLM pages
// ("I-DLM：扩散模型如何用“自省一致性”追上自回归模型质量", section
// "Introspective Strided Decoding（ISD）"; "自省扩散语言模型的 token 生成机制与
// 工程实践", section "从质量差距到自省机制"): p is the anchor distribution of the
// clean slot one position earlier (logit shift), q the proposal distribution
// of the MASK slot that proposed the token in the previous step.  Proposals
// are argmax ("服务部署与 SGLang 集成": argmax proposal strategy) unless sample
// mode is selected.  A rejection draws its replacement from max(0, p - q), the
// rule under which the pages' "lossless" claim holds.
//
// All reductions run in a fixed order (no floating-point atomics), so a
// repeated call is bit-identical.  Cross-CTA combination uses the
// last-block-done ticket: every CTA publishes its partial, fences, and the
// CTA that draws the last ticket combines; nothing spins.
#include "common.cuh"
#include "launch.h"
#include "plan.h"
#include "sm100.cuh"

namespace isd {

// ---------------------------------------------------------------------------
// a5: per-row max, sum exp(z - max), argmax (ties -> lowest index)
// ---------------------------------------------------------------------------
template <int THREADS>
__global__ void __launch_bounds__(THREADS)
row_stats_kernel(const float* __restrict__ logits, int V, int n_chunks, int chunk_len,
                 float4* __restrict__ part, int* __restrict__ ticket,
                 isd_row_stat* __restrict__ out) {
    const int row = blockIdx.y;
    const int ch = blockIdx.x;
    const int beg = ch * chunk_len;
    const int end = min(V, beg + chunk_len);
    const float* z = logits + (size_t)row * V;
    RowStat st = rowstat_empty();
    if ((V & 3) == 0) {
        for (int i = beg + 4 * threadIdx.x; i < end; i += 4 * THREADS) {
            const float4 v = ld_stream_f4(z + i);
            rowstat_push(st, v.x, i);
            rowstat_push(st, v.y, i + 1);
            rowstat_push(st, v.z, i + 2);
            rowstat_push(st, v.w, i + 3);
        }
    } else {
        for (int i = beg + threadIdx.x; i < end; i += THREADS) rowstat_push(st, __ldg(z + i), i);
    }
    st = rowstat_block_reduce<THREADS>(st);
    if (threadIdx.x != 0) return;
    if (n_chunks == 1) {
        out[row] = isd_row_stat{st.m, st.s, st.idx, 0};
        return;
    }
    part[(size_t)row * n_chunks + ch] = make_float4(st.m, st.s, __int_as_float(st.idx), 0.f);
    __threadfence();
    const int t = atomicAdd(&ticket[row], 1);
    if (t != n_chunks - 1) return;
    __threadfence();
    RowStat acc = rowstat_empty();
    for (int k = 0; k < n_chunks; ++k) {
        const float4 p = __ldcg(&part[(size_t)row * n_chunks + k]);
        acc = rowstat_merge(acc, RowStat{p.x, p.y, __float_as_int(p.z)});
    }
    out[row] = isd_row_stat{acc.m, acc.s, acc.idx, 0};
    ticket[row] = 0;
}

// ---------------------------------------------------------------------------
// a6-a9
// ---------------------------------------------------------------------------
struct AcceptArgs {
    int B, N, V, mode;
    const float* logits;
    const isd_row_stat* stats;
    const float* prev_logits;
    const isd_row_stat* prev_stats;
    const int32_t* n_clean;
    const int32_t* clean_tok;
    const int32_t* kv_len;
    const float* uniforms;
    int32_t* accept_len;
    int32_t* out_tok;
    int32_t* next_n_clean;
    int32_t* next_clean_tok;
    int32_t* next_kv_len;
    float* ratio;
    float* part;     // [B][N+1][n_chunks] chunk totals
    int* ticket;     // [B] tickets, then [B] decided states, then the decided count
    int n_chunks;
    bool vec;        // logits rows 16-byte aligned (V % 4 == 0, aligned bases)
    int32_t* err_flag;
    // inside a whole step: this step's row statistics come as the LM head's
    // partials ([B*Q][n_parts]); the kernel merges the rows it needs and the
    // CTA of chunk 0 writes each request's merged rows to stats_out
    const float4* stats_part;
    int n_parts;
    isd_row_stat* stats_out;
};

// Weight of vocabulary entry i for "row" r of a sweep.
//   sample-mode proposal rows: exp(z_i - max) of that row;
//   residual of a rejecting request: max(0, p_i - q_i), evaluated as
//     q_i * expm1(log p_i - log q_i),
//     log p_i - log q_i = (zp_i - zq_i) + [(mq - mp) + log(Sq / Sp)].
//   A plain difference of the two probabilities cancels catastrophically
//   when p and q nearly agree (both ~1/V, difference ~1e-6 of that); in this
//   form entries with equal logits get exactly equal log-ratios, so the
//   weights keep their shape and only the row constant carries rounding.
struct SweepRow {
    const float* zp;
    const float* zq;  // null for proposal rows
    float mp, mq, inv_sq, k;  // k = (mq - mp) + log(Sq / Sp)
};

// e^d - 1 for d > 0 without cancellation: the Taylor series
// d (1 + d/2 (1 + d/3 (1 + d/4 (1 + d/5)))) below 0.1 (truncation error under
// d^5/720 relative, i.e. < 2e-8), and e^d - 1 directly above it, where the
// subtraction loses at most a factor 1/(1 - e^-d) < 11 of relative precision.
ISD_DEVINL float expm1_pos(float d) {
    if (d < 0.1f) return d * (1.f + 0.5f * d * (1.f + d * (1.f / 3.f) * (1.f + 0.25f * d * (1.f + 0.2f * d))));
    return __expf(d) - 1.f;
}

ISD_DEVINL float weight_of(const SweepRow& r, float zp, float zq) {
    if (!r.zq) return __expf(zp - r.mp);
    const float d = (zp - zq) + r.k;
    if (!(d > 0.f)) return 0.f;
    return __expf(zq - r.mq) * r.inv_sq * expm1_pos(d);
}

constexpr int kSeg = kAcceptChunk / kAcceptThreads;  // contiguous entries per thread
static_assert(kSeg % 4 == 0, "a thread's segment is whole float4s");

// Weights of entries s0 .. s0+kSeg-1 (zero at and past end).  With vec (rows
// 16-byte aligned) a full segment is read as float4s, every load of the
// segment issued before the first is used.
ISD_DEVINL void seg_weights(const SweepRow& r, int s0, int end, bool vec, float (&w)[kSeg]) {
    float zp[kSeg], zq[kSeg];
    if (vec && s0 + kSeg <= end) {
#pragma unroll
        for (int v = 0; v < kSeg / 4; ++v) {
            const float4 t = __ldg(reinterpret_cast<const float4*>(r.zp + s0) + v);
            zp[4 * v] = t.x;
            zp[4 * v + 1] = t.y;
            zp[4 * v + 2] = t.z;
            zp[4 * v + 3] = t.w;
        }
        if (r.zq) {
#pragma unroll
            for (int v = 0; v < kSeg / 4; ++v) {
                const float4 t = __ldg(reinterpret_cast<const float4*>(r.zq + s0) + v);
                zq[4 * v] = t.x;
                zq[4 * v + 1] = t.y;
                zq[4 * v + 2] = t.z;
                zq[4 * v + 3] = t.w;
            }
        }
#pragma unroll
        for (int k = 0; k < kSeg; ++k) w[k] = weight_of(r, zp[k], r.zq ? zq[k] : 0.f);
        return;
    }
#pragma unroll
    for (int k = 0; k < kSeg; ++k) {
        const int i = s0 + k;
        zp[k] = i < end ? __ldg(r.zp + i) : 0.f;
        zq[k] = (i < end && r.zq) ? __ldg(r.zq + i) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kSeg; ++k) w[k] = s0 + k < end ? weight_of(r, zp[k], zq[k]) : 0.f;
}

// Exclusive block scan of one float per thread (fixed order); returns the
// exclusive prefix and writes the block total to *total.
ISD_DEVINL float block_exclusive_scan(float v, float* total) {
    __shared__ float warp_tot[kAcceptThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += n;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    float base = 0.f, tot = 0.f;
#pragma unroll
    for (int w = 0; w < kAcceptThreads / 32; ++w) {
        if (w < warp) base += warp_tot[w];
        tot += warp_tot[w];
    }
    __syncthreads();
    *total = tot;
    return base + incl - v;
}

// Chunk [beg, end): per-thread contiguous segments; returns the chunk total
// (identical bits every time it is recomputed) and, if target >= 0, the first
// index whose prefix exceeds target (or -1).
ISD_DEVINL float chunk_scan(const SweepRow& r, int beg, int end, bool vec, float target,
                            int* found) {
    float w[kSeg];
    const int s0 = beg + threadIdx.x * kSeg;
    seg_weights(r, s0, end, vec, w);
    float local = 0.f;
#pragma unroll
    for (int k = 0; k < kSeg; ++k) local += w[k];
    float total;
    const float excl = block_exclusive_scan(local, &total);
    if (target >= 0.f) {
        __shared__ int first;
        if (threadIdx.x == 0) first = 0x7fffffff;
        __syncthreads();
        if (excl + local > target) atomicMin(&first, (int)threadIdx.x);
        __syncthreads();
        int idx = -1;
        if ((int)threadIdx.x == first) {
            float part = 0.f;
            for (int k = 0; k < kSeg; ++k) {
                part += w[k];
                if (w[k] > 0.f && excl + part > target) {
                    idx = s0 + k;
                    break;
                }
            }
        }
        // last index with positive weight, for the rounding fallback
        __shared__ int last_pos, hit;
        if (threadIdx.x == 0) {
            last_pos = -1;
            hit = -1;
        }
        __syncthreads();
        for (int k = kSeg - 1; k >= 0; --k)
            if (w[k] > 0.f && s0 + k < end) {
                atomicMax(&last_pos, s0 + k);
                break;
            }
        if (idx >= 0) hit = idx;
        __syncthreads();
        *found = hit >= 0 ? hit : last_pos;
        __syncthreads();
    }
    return total;
}

// Emitted tokens and next state of request b (thread 0): state > 0 is the
// rejected proposal index j (the first j - 2 proposals kept, then the draw
// picked[0]); state 0 keeps all c clean tokens and proposes picked[0..N-1].
ISD_DEVINL void emit_request(const AcceptArgs& a, int b, int state, int c, const int* picked) {
    const int N = a.N;
    const int* tok = a.clean_tok + (size_t)b * N;
    int32_t* ot = a.out_tok + (size_t)b * N;
    int32_t* nt = a.next_clean_tok + (size_t)b * N;
    int A;
    if (state > 0) {
        A = state - 1;
        for (int k = 0; k < A - 1; ++k) ot[k] = tok[k + 1];
        ot[A - 1] = picked[0];
        for (int k = A; k < N; ++k) ot[k] = -1;
        nt[0] = picked[0];
        for (int k = 1; k < N; ++k) nt[k] = -1;
        a.next_n_clean[b] = 1;
    } else {
        A = c;
        for (int k = 0; k < c - 1; ++k) ot[k] = tok[k + 1];
        ot[c - 1] = picked[0];
        for (int k = c; k < N; ++k) ot[k] = -1;
        for (int k = 0; k < N; ++k) nt[k] = picked[k];
        a.next_n_clean[b] = N;
    }
    a.accept_len[b] = A;
    a.next_kv_len[b] = a.kv_len[b] + A;
}

// One CTA per (sweep item) slot, B x n_chunks in all.  CTAs 0 .. B-1 decide
// the requests (merging every row of theirs, written to stats_out in fused
// mode), write the ratios and, when a request draws nothing, its outputs;
// then each counts itself in `decided`.  Every CTA waits (bounded) until all
// B are decided and takes the item of its index among the chunks of the
// requests that draw (a rejection's residual, or sample-mode proposals), in
// request order; the CTAs past them leave at once.  The CTA holding a
// request's last ticket scans its chunk totals in chunk order and draws.
// Decisions and draws do not depend on which CTA computes them, so a
// repeated call is bit-identical.
__global__ void __launch_bounds__(kAcceptThreads, kAcceptMinBlocks)
accept_kernel(const __grid_constant__ AcceptArgs a) {
    pdl_trigger();
    pdl_wait();
    const int cta = blockIdx.x;
    const int N = a.N, Q = 2 * N - 1, V = a.V;
    const int rcols = N > 1 ? N - 1 : 1;
    const bool fused = a.stats_part != nullptr;
    int* req_state = a.ticket + a.B;
    int* decided = a.ticket + 2 * a.B;
    __shared__ int s_last, s_bad, s_b, s_ok;
    __shared__ float s_ratio[16];
    __shared__ isd_row_stat s_stats[32];  // the decided request's merged rows (Q <= 31)
    __shared__ int picked[16];            // N <= 16 (checked on the host); written by thread 0
    // this step's statistics of row k of request b outside the decision:
    // merged by the decider (stats_out, read from L2), or given
    auto stat_of = [&](int b, int k) -> isd_row_stat {
        if (!fused) return a.stats[(size_t)b * Q + k];
        const float4 v = __ldcg(reinterpret_cast<const float4*>(a.stats_out + (size_t)b * Q + k));
        return isd_row_stat{v.x, v.y, __float_as_int(v.z), __float_as_int(v.w)};
    };

    // ------------------------------------------------------------ decisions
    if (cta < a.B) {
        const int b = cta;
        const float* ub = a.uniforms + (size_t)b * 2 * N;
        const int c_in = __ldg(&a.n_clean[b]);
        const bool bad_c = (c_in < 1 || c_in > N);
        if (threadIdx.x == 0) s_bad = 0;
        __syncthreads();
        // the gathered p/q operands of every tested proposal (one round of
        // loads, in flight while the row statistics are merged)
        const int jt = (int)threadIdx.x + 2;
        float zp = 0.f, zq = 0.f;
        isd_row_stat sq = isd_row_stat{0.f, 1.f, 0, 0};
        bool have = false;
        if (!bad_c && jt <= c_in) {
            const int x = __ldg(&a.clean_tok[(size_t)b * N + jt - 1]);
            if (x < 0 || x >= V) {
                s_bad = 1;
            } else {
                const size_t rp = (size_t)b * Q + (jt - 2);
                const size_t rq = (size_t)b * Q + (N + jt - 2);
                zp = a.logits[rp * V + x];
                zq = a.prev_logits[rq * V + x];
                sq = a.prev_stats[rq];
                have = true;
            }
        }
        // every row of the request: merged here (one warp per row) and
        // written out, or given
        const int wid = (int)threadIdx.x >> 5;
        for (int k = wid; k < Q; k += kAcceptThreads / 32) {
            isd_row_stat v;
            if (fused) {
                const RowStat st = warp_merge_partials<8>(a.stats_part + ((size_t)b * Q + k) * a.n_parts, a.n_parts);
                v = isd_row_stat{st.m, st.s, st.idx, 0};
                if ((threadIdx.x & 31) == 0) {
                    a.stats_out[(size_t)b * Q + k] = v;
                    __threadfence();  // before the decision is counted
                }
            } else {
                v = a.stats[(size_t)b * Q + k];
            }
            if ((threadIdx.x & 31) == 0) s_stats[k] = v;
        }
        __syncthreads();
        // p(x)/q(x) = exp((zp - mp) - (zq - mq)) * Sq / Sp
        if (have) {
            const isd_row_stat sp = s_stats[jt - 2];
            s_ratio[jt - 2] = expf((zp - sp.max) - (zq - sq.max)) * (sq.sumexp / sp.sumexp);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int state = 0;
            if (bad_c) {
                raise_flag(a.err_flag, ISD_FLAG_NCLEAN_RANGE);
                state = -1;
            } else if (s_bad) {
                raise_flag(a.err_flag, ISD_FLAG_TOKEN_OOB);
                state = -1;
            } else {
                // the first rejection stops the pass
                for (int j = 2; j <= c_in; ++j)
                    if (!(ub[j - 2] < s_ratio[j - 2])) {
                        state = j;
                        break;
                    }
            }
            if (a.ratio) {
                const int tested = state > 0 ? state - 1 : (state == 0 ? c_in - 1 : 0);
                for (int k = 0; k < rcols; ++k)
                    a.ratio[(size_t)b * rcols + k] = k < tested ? s_ratio[k] : -1.f;
            }
            if (state < 0) {  // invalid request: emit nothing, carry the state over
                const int* tok = a.clean_tok + (size_t)b * N;
                a.accept_len[b] = 0;
                a.next_n_clean[b] = c_in;
                a.next_kv_len[b] = a.kv_len[b];
                for (int k = 0; k < N; ++k) {
                    a.out_tok[(size_t)b * N + k] = -1;
                    a.next_clean_tok[(size_t)b * N + k] = tok[k];
                }
            } else if (state == 0 && a.mode != ISD_PROPOSE_SAMPLE) {
                // every proposal kept, argmax proposals: nothing to draw
                picked[0] = s_stats[c_in - 1].argmax;
                for (int m = 0; m + 1 < N; ++m) picked[m + 1] = s_stats[N + m].argmax;
                emit_request(a, b, 0, c_in, picked);
            }
            req_state[b] = state;
            __threadfence();
            asm volatile("red.release.gpu.global.add.s32 [%0], 1;\n" ::"l"(decided) : "memory");
        }
    }

    // ------------------------------------------------------------ draws
    if (threadIdx.x == 0) {
        // bounded wait until every request is decided (the deciders are the
        // first B CTAs of the grid; they wait for nothing)
        int ok = 0;
        const uint64_t t0 = sm100::global_ns();
        for (uint32_t it = 0;; ++it) {
            int v;
            asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(decided) : "memory");
            if (v >= a.B) {
                ok = 1;
                break;
            }
            if ((it & 63) == 63 && sm100::global_ns() - t0 > 2000000000ull) {
                raise_flag(a.err_flag, ISD_FLAG_WAIT_TIMEOUT);
                break;
            }
        }
        s_ok = ok;
        s_b = -1;
    }
    __syncthreads();
    if (!s_ok) return;
    // this CTA's item: request number cta / n_chunks among those that draw
    const int r_idx = cta / a.n_chunks, ch = cta - r_idx * a.n_chunks;
    {
        int base = 0;
        for (int t0 = 0; t0 < a.B && base <= r_idx; t0 += kAcceptThreads) {
            const int t = t0 + (int)threadIdx.x;
            int f = 0;
            if (t < a.B) {
                const int st = __ldcg(req_state + t);
                f = st > 0 || (st == 0 && a.mode == ISD_PROPOSE_SAMPLE);
            }
            float tot;
            const int excl = base + (int)block_exclusive_scan((float)f, &tot);
            if (f && excl == r_idx) s_b = t;
            base += (int)tot;
            __syncthreads();
        }
    }
    __syncthreads();
    const int b = s_b;
    if (b < 0) return;  // past the drawing requests' chunks
    const int state = __ldcg(req_state + b);
    const int c = __ldg(&a.n_clean[b]);
    const int nrows = state > 0 ? 1 : N;
    const float* ub = a.uniforms + (size_t)b * 2 * N;
    // the inverse-CDF rows of request b: the residual max(0, p - q) of the
    // rejected proposal, or (sample mode) the N proposal rows
    auto row_of = [&](int k, SweepRow* r) {
        if (state > 0) {
            const size_t rp = (size_t)b * Q + (state - 2);
            const size_t rq = (size_t)b * Q + (N + state - 2);
            const isd_row_stat sp = stat_of(b, state - 2), sq = a.prev_stats[rq];
            *r = SweepRow{a.logits + rp * V, a.prev_logits + rq * V, sp.max, sq.max,
                          1.f / sq.sumexp, (sq.max - sp.max) + logf(sq.sumexp / sp.sumexp)};
        } else {
            const size_t rr = (size_t)b * Q + (k == 0 ? c - 1 : N + k - 1);
            const isd_row_stat st = stat_of(b, k == 0 ? c - 1 : N + k - 1);
            *r = SweepRow{a.logits + rr * V, nullptr, st.max, 0.f, 0.f, 0.f};
        }
    };
    float* part = a.part + (size_t)b * (N + 1) * a.n_chunks;
    {
        const int beg = ch * kAcceptChunk, end = min(V, beg + kAcceptChunk);
        for (int k = 0; k < nrows; ++k) {
            SweepRow r;
            row_of(k, &r);
            int dummy;
            const float tot = chunk_scan(r, beg, end, a.vec, -1.f, &dummy);
            if (threadIdx.x == 0) part[(size_t)k * a.n_chunks + ch] = tot;
        }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&a.ticket[b], 1) == a.n_chunks - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int k = 0; k < nrows; ++k) {
        SweepRow r;
        row_of(k, &r);
        const float u = state > 0 ? ub[N - 1] : ub[N + k];
        // chunk totals in chunk order, scanned by the whole block
        __shared__ float s_target;
        __shared__ int s_chunk, s_hit, s_lastpos;
        const float tv = (int)threadIdx.x < a.n_chunks
                             ? __ldcg(&part[(size_t)k * a.n_chunks + threadIdx.x]) : 0.f;
        float total;
        const float excl = block_exclusive_scan(tv, &total);
        const float target = u * total;
        if (threadIdx.x == 0) {
            s_hit = 0x7fffffff;
            s_lastpos = -1;
        }
        __syncthreads();
        if (tv > 0.f) atomicMax(&s_lastpos, (int)threadIdx.x);
        if ((int)threadIdx.x < a.n_chunks && excl + tv > target) atomicMin(&s_hit, (int)threadIdx.x);
        __syncthreads();
        if (threadIdx.x == 0) {
            if (!(total > 0.f)) {
                s_chunk = -2;  // no mass: residual falls back to argmax p
                s_target = 0.f;
            } else if (s_hit == 0x7fffffff) {
                s_chunk = s_lastpos;
                s_target = 3.0e38f;  // take the last positive entry of that chunk
            } else {
                s_chunk = s_hit;
            }
        }
        __syncthreads();
        if (s_chunk >= 0 && s_chunk == s_hit && (int)threadIdx.x == s_hit)
            s_target = fmaxf(target - excl, 0.f);
        __syncthreads();
        const int q = s_chunk;
        const float tgt = s_target;
        __syncthreads();
        int y;
        if (q == -2) {  // argmax of the anchor (or proposal) row
            y = stat_of(b, state > 0 ? state - 2 : (k == 0 ? c - 1 : N + k - 1)).argmax;
        } else {
            const int beg2 = q * kAcceptChunk, end2 = min(V, beg2 + kAcceptChunk);
            chunk_scan(r, beg2, end2, a.vec, tgt, &y);
        }
        if (threadIdx.x == 0) picked[k] = y;
    }
    if (threadIdx.x == 0) {
        emit_request(a, b, state, c, picked);
        a.ticket[b] = 0;
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_row_stats(const Plan& p, const float* logits, int rows, int V,
                             isd_row_stat* out, void* ws, cudaStream_t st) {
    char* w = static_cast<char*>(ws);
    dim3 grid(p.stats_chunks, rows);
    row_stats_kernel<kStatsThreads><<<grid, kStatsThreads, 0, st>>>(
        logits, V, p.stats_chunks, p.stats_chunk_len,
        reinterpret_cast<float4*>(w + p.off_stats_part),
        reinterpret_cast<int*>(w + p.off_stats_ticket), out);
    return cudaGetLastError();
}

cudaError_t launch_accept(const Plan& p, const isd_dims* d, const float* logits,
                          const isd_row_stat* stats, const float* prev_logits,
                          const isd_row_stat* prev_stats, const int32_t* n_clean,
                          const int32_t* clean_tok, const int32_t* kv_len, const float* uniforms,
                          int32_t* accept_len, int32_t* out_tok, int32_t* next_n_clean,
                          int32_t* next_clean_tok, int32_t* next_kv_len, float* ratio, void* ws,
                          int32_t* err_flag, cudaStream_t st, bool pdl, const float4* stats_part,
                          int n_parts, isd_row_stat* stats_out) {
    char* w = static_cast<char*>(ws);
    AcceptArgs a;
    a.stats_part = stats_part;
    a.n_parts = n_parts;
    a.stats_out = stats_out;
    a.B = d->B;
    a.N = d->N;
    a.V = d->V;
    a.mode = d->proposal_mode;
    a.logits = logits;
    a.stats = stats;
    a.prev_logits = prev_logits;
    a.prev_stats = prev_stats;
    a.n_clean = n_clean;
    a.clean_tok = clean_tok;
    a.kv_len = kv_len;
    a.uniforms = uniforms;
    a.accept_len = accept_len;
    a.out_tok = out_tok;
    a.next_n_clean = next_n_clean;
    a.next_clean_tok = next_clean_tok;
    a.next_kv_len = next_kv_len;
    a.ratio = ratio;
    a.part = reinterpret_cast<float*>(w + p.off_acc_part);
    a.ticket = reinterpret_cast<int*>(w + p.off_acc_ticket);
    a.n_chunks = p.acc_chunks;
    a.vec = d->V % 4 == 0 && reinterpret_cast<uintptr_t>(logits) % 16 == 0 &&
            reinterpret_cast<uintptr_t>(prev_logits) % 16 == 0;
    a.err_flag = err_flag;
    dim3 grid(d->B * p.acc_chunks);
    return launch_kernel(pdl, accept_kernel, grid, dim3(kAcceptThreads), 0, st, a);
}

}  // namespace isd
