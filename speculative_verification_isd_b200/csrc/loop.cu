// Device-resident stationary-batch decode loop: n ISD steps enqueued back to
// back with every piece of per-step bookkeeping on the device, so a host
// thread issues the whole loop (or captures it once into a CUDA graph) and
// reads nothing until the end.
//
// The serving notes of the I-DLM pages credit two engine features with much
// of the measured throughput: a stationary batch in which every request
// advances independently, without synchronising on the batch
// ("自省扩散语言模型的 token 生成机制与工程实践", section "服务部署与 SGLang 集成";
// I-DLM project page, the paragraph on requests advancing independently), and
// CUDA-graph capture of the decode loop (same section).  Here each step
//   1. builds the block's activations from each request's state: the clean
//      slots hold that request's tokens, the MASK slots (and inactive clean
//      slots) the MASK token, and the per-layer forward is stood in for by a
//      token -> (q, k, v) table lookup (the pages give no layer internals);
//   2. grows each request's page list so it covers kv_len + 2N-1 positions,
//      taking pages from a bump allocator in request order (deterministic);
//   3. runs the ISD step (attention, LM head, accept) on the state buffers
//      of this step, writing the next state into the other buffer of each
//      pair, and its logits / row statistics into the buffer the next step
//      reads as the previous step's.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "launch.h"
#include "plan.h"

namespace isd {

struct PrepArgs {
    int B, N, Q, Hq, Hkv, D, V, P, num_pages, max_pages;
    const uint16_t* Eq;  // [V+1, Hq, D]
    const uint16_t* Ek;  // [V+1, Hkv, D]
    const uint16_t* Ev;
    const int32_t* n_clean;    // null: the N first slots are all clean slots (c = N)
    const int32_t* clean_tok;
    int mask_neg;              // 1: a negative token is an uncommitted position (MASK row)
    const float2* rope;        // [rope_len][D/2] (cos, sin), or null: no rotation
    int rope_len;
    const int32_t* kv_len;
    int32_t* page_table;
    int32_t* pages_used;
    int32_t* next_free;
    uint16_t* q;
    uint16_t* k_new;
    uint16_t* v_new;
    int32_t* err_flag;
};

constexpr int kPrepThreads = 256;

// Rotary embedding of one 8-pair piece of a head vector: lo holds elements
// 8j..8j+7 of the first half, hi the same elements of the second half (pairs
// (i, i + D/2)); each product and sum is rounded separately (no contraction),
// then the result is rounded once to bf16.
ISD_DEVINL void rope_rotate8(const uint4& lo, const uint4& hi, const float2* cs, uint4& olo,
                             uint4& ohi) {
    const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&lo);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hi);
    __nv_bfloat162* ol = reinterpret_cast<__nv_bfloat162*>(&olo);
    __nv_bfloat162* oh = reinterpret_cast<__nv_bfloat162*>(&ohi);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(l2[e]), y = __bfloat1622float2(h2[e]);
        const float2 c0 = __ldg(cs + 2 * e), c1 = __ldg(cs + 2 * e + 1);
        const float xl0 = __fsub_rn(__fmul_rn(x.x, c0.x), __fmul_rn(y.x, c0.y));
        const float yh0 = __fadd_rn(__fmul_rn(y.x, c0.x), __fmul_rn(x.x, c0.y));
        const float xl1 = __fsub_rn(__fmul_rn(x.y, c1.x), __fmul_rn(y.y, c1.y));
        const float yh1 = __fadd_rn(__fmul_rn(y.y, c1.x), __fmul_rn(x.y, c1.y));
        ol[e] = __floats2bfloat162_rn(xl0, xl1);
        oh[e] = __floats2bfloat162_rn(yh0, yh1);
    }
}

// One table row (id) of nh heads -> dst, rotated by position pos when cs
// (that position's table row) is given, else copied.
ISD_DEVINL void prep_rows(const uint16_t* table, int id, int nh, int D, uint16_t* dst_row,
                          const float2* cs) {
    const uint4* src = reinterpret_cast<const uint4*>(table + (size_t)id * nh * D);
    uint4* dst = reinterpret_cast<uint4*>(dst_row);
    if (!cs) {
        for (int i = threadIdx.x; i < nh * D / 8; i += kPrepThreads) dst[i] = __ldg(src + i);
        return;
    }
    const int halves = D / 16;  // 16-byte pieces in half a head vector
    for (int i = threadIdx.x; i < nh * halves; i += kPrepThreads) {
        const int h = i / halves, j = i - h * halves;
        const uint4* sh = src + (size_t)h * (D / 8);
        uint4* dh = dst + (size_t)h * (D / 8);
        rope_rotate8(__ldg(sh + j), __ldg(sh + j + halves), cs + 8 * j, dh[j], dh[j + halves]);
    }
}

// grid (Q, B): block slot s of request b copies its table rows (16 bytes per
// thread); CTA (0, 0) also extends every request's page list, in request
// order, from the bump allocator.
__global__ void __launch_bounds__(kPrepThreads) prepare_block_kernel(const __grid_constant__ PrepArgs a) {
    pdl_trigger();
    pdl_wait();  // the state was written by the previous step's accept
    const int s = blockIdx.x, b = blockIdx.y;
    const int c = a.n_clean ? a.n_clean[b] : a.N;
    int id = a.V;  // the MASK row
    if (s < a.N && s < c && c <= a.N) {
        const int t = a.clean_tok[(size_t)b * a.N + s];
        if (t >= 0 && t < a.V) id = t;
        else if (!(a.mask_neg && t < 0) && threadIdx.x == 0) raise_flag(a.err_flag, ISD_FLAG_TOKEN_OOB);
    }
    const size_t row = (size_t)b * a.Q + s;
    // rotary embedding (the block of N rows at kv_len .. kv_len+N-1 only)
    const float2* cs = nullptr;
    if (a.rope) {
        const int pos = max(a.kv_len[b], 0) + s;
        if (pos < a.rope_len) cs = a.rope + (size_t)pos * (a.D / 2);
        else if (threadIdx.x == 0) raise_flag(a.err_flag, ISD_FLAG_CAPACITY);
    }
    prep_rows(a.Eq, id, a.Hq, a.D, a.q + row * a.Hq * a.D, cs);
    prep_rows(a.Ek, id, a.Hkv, a.D, a.k_new + row * a.Hkv * a.D, cs);
    prep_rows(a.Ev, id, a.Hkv, a.D, a.v_new + row * a.Hkv * a.D, nullptr);
    if (s != 0 || b != 0) return;
    // page bookkeeping: request r needs ceil((kv_len + Q) / P) pages (at most
    // the table's width); new pages are handed out in request order
    __shared__ int warp_sum[kPrepThreads / 32];
    __shared__ int s_base;
    if (threadIdx.x == 0) s_base = *a.next_free;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int r0 = 0; r0 < a.B; r0 += kPrepThreads) {
        const int r = r0 + (int)threadIdx.x;
        int have = 0, add = 0;
        if (r < a.B) {
            const long long want = ((long long)max(a.kv_len[r], 0) + a.Q + a.P - 1) / a.P;
            have = a.pages_used[r];
            const int need = (int)min(want, (long long)a.max_pages);
            add = need > have ? need - have : 0;
            if (want > a.max_pages) raise_flag(a.err_flag, ISD_FLAG_CAPACITY);
        }
        // exclusive scan of add over the block, in request order
        int incl = add;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        if (lane == 31) warp_sum[warp] = incl;
        __syncthreads();
        int base = s_base, total = 0;
        for (int w = 0; w < kPrepThreads / 32; ++w) {
            if (w < warp) base += warp_sum[w];
            total += warp_sum[w];
        }
        const int first = base + incl - add;
        if (r < a.B && add > 0) {
            int got = 0;
            for (int i = 0; i < add; ++i) {
                const int page = first + i;
                if (page >= a.num_pages) {
                    raise_flag(a.err_flag, ISD_FLAG_CAPACITY);
                    break;
                }
                a.page_table[(size_t)r * a.max_pages + have + i] = page;
                ++got;
            }
            a.pages_used[r] = have + got;
        }
        __syncthreads();
        if (threadIdx.x == 0) s_base += total;
        __syncthreads();
    }
    if (threadIdx.x == 0) *a.next_free = min(s_base, a.num_pages);
}

// Q: block slots per request (2N - 1 for an ISD block; N for an SDAR block,
// whose tokens come with n_clean null and mask_neg set, and whose q and k
// rows may be rotated by position: rope [rope_len][D/2] (cos, sin) or null).
cudaError_t launch_prepare_block(const isd_dims* d, int Q, const uint16_t* Eq, const uint16_t* Ek,
                                 const uint16_t* Ev, const int32_t* n_clean, const int32_t* clean_tok,
                                 bool mask_neg, const float* rope, int rope_len,
                                 const int32_t* kv_len, int32_t* page_table,
                                 int32_t* pages_used, int32_t* next_free, uint16_t* q,
                                 uint16_t* k_new, uint16_t* v_new, int32_t* err_flag,
                                 cudaStream_t st, bool pdl) {
    PrepArgs a;
    a.B = d->B;
    a.N = d->N;
    a.Q = Q;
    a.Hq = d->Hq;
    a.Hkv = d->Hkv;
    a.D = d->D;
    a.V = d->V;
    a.P = d->page_size;
    a.num_pages = d->num_pages;
    a.max_pages = d->max_pages_per_req;
    a.Eq = Eq;
    a.Ek = Ek;
    a.Ev = Ev;
    a.n_clean = n_clean;
    a.clean_tok = clean_tok;
    a.mask_neg = mask_neg ? 1 : 0;
    a.rope = reinterpret_cast<const float2*>(rope);
    a.rope_len = rope_len;
    a.kv_len = kv_len;
    a.page_table = page_table;
    a.pages_used = pages_used;
    a.next_free = next_free;
    a.q = q;
    a.k_new = k_new;
    a.v_new = v_new;
    a.err_flag = err_flag;
    return launch_kernel(pdl, prepare_block_kernel, dim3(a.Q, a.B), dim3(kPrepThreads), 0, st, a);
}

}  // namespace isd
