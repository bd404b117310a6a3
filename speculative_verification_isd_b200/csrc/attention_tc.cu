// Strict-causal GQA attention over the paged KV cache (a2) on the
// 5th-generation tensor cores, with the KV append (a1) as a separate kernel.
//
// Same operation as attention.cu: every query slot of the block attends to
// the cached prefix and to the block keys at or before its own position
// (strict causal mask over clean and MASK slots, "I-DLM：扩散模型如何用“自省一致性”
// 追上自回归模型质量", section "三项关键训练创新"; paged KV cache, section
// "推理：复用 AR 推理栈").  Organised for sm_100a:
//
//  * kv_append_kernel first writes the block's K/V rows into their pages, so
//    every key is then read from the pool by TMA: a 4-D tensor map (d, kv head,
//    token in page, page) whose page coordinate comes from the page table; a
//    page past the request (or a bad page id) is a box out of range and
//    reads zeros;
//  * the work is split tile-granularly ("stream-K"): the flattened sequence of
//    (request, kv head, 128-key tile) is cut into G equal ranges, one per
//    persistent CTA, so every SM streams the same number of KV bytes.  A
//    (request, kv head) cut by a range boundary leaves a partial result per
//    CTA; the CTA that draws the last ticket merges them in CTA order, so the
//    result does not depend on timing;
//  * K and V halves of a stage have their own ring barriers and their own
//    TMA producer warp: the K half is refilled as soon as S = K.Q^T has
//    read it, the V half after P.V, so a stage's bytes wait in shared memory
//    only about one product's latency (with a 3-stage ring of 128 keys,
//    holding a stage for the whole S -> softmax -> P.V chain measured about
//    3% slower for the whole step at B=32, N=4);
//  * per 128-key tile two tensor-core products, issued by one thread:
//      S^T[128 keys, R rows] = K . Q^T         (M=128, N=R, K=128 d)
//      O^T[128 d,   R rows] += V^T . P^T       (M=128, N=R, K=128 keys)
//    with Q/K/V/P in 128-byte-swizzled shared memory and S, O in TMEM;
//  * softmax warps own one key each per thread and 16 of the rows (32 at
//    R = 64; R / RC groups of 4 warps); the
//    per-row reference maximum moves only when a score exceeds it by more
//    than 2^8 (then O^T is rescaled in TMEM), and P^T goes to shared memory
//    as bf16 for the second product;
//  * every wait is bounded (about 2 s): on time-out the CTA raises
//    ISD_FLAG_WAIT_TIMEOUT, all roles leave their loops, in-flight copies and
//    MMAs are drained and TMEM is released.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "plan.h"
#include "sm100.cuh"
#include "launch.h"
#include "tmap.h"

namespace isd {

void set_error_detail(const char* msg);

namespace {

constexpr int kTcKeys = 128;            // keys per tile (M of S^T)
// A (request, kv head) also costs an epilogue: the partition counts it as
// this many extra tiles, so CTAs whose ranges hold many short requests get
// fewer tiles.
constexpr int kTcUnitCost = 4;
constexpr int kTcHalf = kTcKeys * 128;  // bytes of one 64-d half of a K or V tile
constexpr uint64_t kTcWaitNs = 2000000000ull;
// K and V ring depths (stages of 128 keys) when shared memory allows: a K
// half is held only until its S product completes, a V half until its P.V
// product, after the softmax of the tile
constexpr int kTcDeepK = 3, kTcDeepV = 3;

struct TcArgs {
    int B, N, Q, Hq, Hkv, grp, rows, P, num_pages, max_pages;
    float scale_log2;
    const int32_t* page_table;
    const int32_t* kv_len;
    const int32_t* n_clean;  // null: every one of the N first slots is active (c = N)
    int bidir;          // 1: every row sees the whole block (block-causal mask)
    __nv_bfloat16* out;
    float* part;        // [gridDim.x][2][part_stride] partial results
    int part_stride;    // floats per partial: R maxima, R sums, R x 128 O values
    int* ticket;        // [B * Hkv], zero between calls
    int* part_flag;     // [gridDim.x][2]: partial written (cleared by the KV append and by its reader)
    int32_t* err_flag;
};

ISD_DEVINL int tc_slot_pos(int s, int kv, int c, int N) {
    if (s < c) return kv + s;
    if (s < N) return -1;
    return kv + c + (s - N);
}

ISD_DEVINL int tc_clean(const TcArgs& a, int b) { return a.n_clean ? a.n_clean[b] : a.N; }

// Keys of request b (prefix and active block rows: c clean slots, then the
// Q - N slots after them); 0 for a request that cannot be served (bad
// n_clean, negative or over-capacity length).
ISD_DEVINL int tc_total_keys(const TcArgs& a, int b) {
    const int kv = a.kv_len[b], c = tc_clean(a, b);
    if (c < 1 || c > a.N || kv < 0) return 0;
    const long long t = (long long)kv + c + a.Q - a.N;
    if ((t + a.P - 1) / a.P > a.max_pages) return 0;
    return (int)t;
}

// a1: one CTA per (request, block position): that position's K and V rows
// for all kv heads go into their page, 16 bytes per thread.  The CTA of block
// position 0 also clears the request's attention counters (and, if given, one
// more counter per request for the kernels that follow), and writes zero
// attention output for a request that cannot be served; CTA (0, 0) clears
// clear_count more counters at clear_range (for later kernels of the step).
__global__ void kv_append_kernel(TcArgs a, const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                                 __nv_bfloat16* k_pool, __nv_bfloat16* v_pool, int* clear_extra,
                                 int* clear_range, int clear_count) {
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x, r = blockIdx.y;
    if (b == 0 && r == 0) {
        if (clear_range)
            for (int i = threadIdx.x; i < clear_count; i += blockDim.x) clear_range[i] = 0;
        for (int i = threadIdx.x; i < 2 * kMaxSMs; i += blockDim.x) a.part_flag[i] = 0;
    }
    const int kv = a.kv_len[b], c = tc_clean(a, b);
    const bool bad_c = (c < 1 || c > a.N);
    const long long want = bad_c ? 0 : (long long)kv + c + a.Q - a.N;
    const bool over = kv < 0 || (want + a.P - 1) / a.P > a.max_pages;
    if (r == 0) {
        for (int i = threadIdx.x; i < a.Hkv; i += blockDim.x) a.ticket[b * a.Hkv + i] = 0;
        if (clear_extra && threadIdx.x == 0) {
            clear_extra[b] = 0;  // accept ticket
            if (b == 0) clear_extra[2 * a.B] = 0;  // accept decided count
        }
    }
    if (bad_c || over) {
        if (r == 0) {
            if (threadIdx.x == 0) raise_flag(a.err_flag, bad_c ? ISD_FLAG_NCLEAN_RANGE : ISD_FLAG_CAPACITY);
            uint4* o = reinterpret_cast<uint4*>(a.out + (size_t)b * a.Q * a.Hq * 128);
            for (int i = threadIdx.x; i < a.Q * a.Hq * 16; i += blockDim.x) o[i] = make_uint4(0, 0, 0, 0);
        }
        return;
    }
    if (r >= c + a.Q - a.N) return;  // block positions: c clean slots, then the Q - N after them
    const int t = kv + r;
    const int slot = r < c ? r : a.N + (r - c);
    const int page = a.page_table[(size_t)b * a.max_pages + t / a.P];
    if (page < 0 || page >= a.num_pages) {
        if (threadIdx.x == 0) raise_flag(a.err_flag, ISD_FLAG_PAGE_OOB);
        return;
    }
    const size_t dst = ((size_t)page * a.P + t % a.P) * a.Hkv * 128;
    const size_t src = ((size_t)b * a.Q + slot) * a.Hkv * 128;
    for (int i = threadIdx.x; i < a.Hkv * 16; i += blockDim.x) {
        *reinterpret_cast<uint4*>(k_pool + dst + (size_t)i * 8) =
            *reinterpret_cast<const uint4*>(k_new + src + (size_t)i * 8);
        *reinterpret_cast<uint4*>(v_pool + dst + (size_t)i * 8) =
            *reinterpret_cast<const uint4*>(v_new + src + (size_t)i * 8);
    }
}

template <int KS, int VS>
struct TcShared {
    uint64_t k_full[KS], k_empty[KS], v_full[VS], v_empty[VS];
    uint64_t s_full[2], s_empty[2], p_full, p_empty;
    uint64_t o_full, o_empty, q_full[2], q_empty[2], drain;
    uint32_t tmem;
    int abort_flag;
    int never;
};

// A CTA's share of one (request, kv head) unit: tiles [t0, t1) of unit u,
// whose position on the partition axis starts at us.
struct TcPiece {
    int u, us, t0, t1, b, g;
};

// Softmax warps: 4 per column group (one per TMEM lane quarter); each
// column group covers RC of the R query rows, so a thread holds RC scores,
// reference maxima and row sums.  RC = 16 (two groups at R = 32: every SM
// sub-partition runs two softmax warps that hide each other's latencies);
// at R = 64, RC = 32 (two groups of 320 threads measured 9% faster than four
// groups of 576, whose registers per thread are too few).
//
// Warpgroup 0 holds the other roles: warp 0 the K/Q TMA producer, warp 1 the
// MMA issuer, warp 2 the V TMA producer (warp 3 idles); the softmax warps are
// warps 4 .. 4 + 4 CG - 1.  With two column groups (384 threads, at most 168
// registers a thread at launch) warpgroup 0 gives registers to the softmax
// warpgroups: kRegsLow x 128 + kRegsHigh x 256 = 384 x 168.
template <int R>
struct TcRoles {
    static constexpr int RC = R == 64 ? 32 : 16;  // rows per softmax thread
    static constexpr int CG = R / RC;           // column groups
    static constexpr int kSoft = 128 * CG;      // softmax threads
    static constexpr int kVWarp = 2;
    static constexpr int kSoftWarp0 = 4;
    static constexpr int kThreads = 128 + kSoft;
    static constexpr bool kRegSplit = R == 64;  // R = 32 fits in 168 registers
    static constexpr int kLaunchRegs = 168;
    static constexpr int kRegsLow = 88, kRegsHigh = 208;
    static_assert(!kRegSplit || kRegsLow * 128 + kRegsHigh * kSoft <= kLaunchRegs * kThreads,
                  "register split exceeds the launch allocation");
};

template <int R, int KS, int VS>
constexpr size_t tc_smem_fixed() {
    return (size_t)(KS + VS) * 2 * kTcHalf  // K and V stages
           + 2 * 2 * R * 128               // Q, two buffers of two 64-d halves
           + 2 * R * 128                   // P^T (two 64-key halves); output staging
           + 4 * R * 4 * 2                 // per-warp row maxima and row sums
           + R * 4                         // per-row causal key limit
           + sizeof(TcShared<KS, VS>);
}
// plus, per launch: 3 ints per request (kv_len, n_clean, keys) and
// B * Hkv + 1 ints of unit offsets on the partition axis

// named barrier 1 over the NT softmax threads, OR of a predicate
template <int NT>
ISD_DEVINL bool group_or(bool v) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, %2, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(NT)
        : "memory");
    return r != 0;
}
template <int NT>
ISD_DEVINL void group_sync() { asm volatile("bar.sync 1, %0;\n" ::"n"(NT) : "memory"); }

template <int C>
ISD_DEVINL void tmem_load_cols(uint32_t taddr, uint32_t (&v)[C]) {
#pragma unroll
    for (int j = 0; j < C / 16; ++j) sm100::tmem_ld16(taddr + j * 16, v + j * 16);
}
template <int C>
ISD_DEVINL void tmem_store_cols(uint32_t taddr, const uint32_t (&v)[C]) {
#pragma unroll
    for (int j = 0; j < C / 16; ++j) sm100::tmem_st16(taddr + j * 16, v + j * 16);
}

template <int R, int KS, int VS>
__global__ void __launch_bounds__(TcRoles<R>::kThreads, 1)
attention_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ TcArgs a) {
    using namespace sm100;
    constexpr int RC = TcRoles<R>::RC, CG = TcRoles<R>::CG, kSoft = TcRoles<R>::kSoft;
    constexpr int kThreads = TcRoles<R>::kThreads;
    constexpr uint32_t kQBytes = 2 * R * 128;
    constexpr uint32_t kPBytes = 2 * R * 128;
    constexpr uint32_t kTmemCols = 4 * R <= 32 ? 32 : (4 * R <= 64 ? 64 : (4 * R <= 128 ? 128 : 256));
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* sK = smem;
    unsigned char* sV = sK + KS * 2 * kTcHalf;
    unsigned char* sQ = sV + VS * 2 * kTcHalf;  // two buffers
    unsigned char* sP = sQ + 2 * kQBytes;
    float* red_m = reinterpret_cast<float*>(sP + kPBytes);   // [4][R]
    float* red_l = red_m + 4 * R;                             // [4][R]
    int* lim = reinterpret_cast<int*>(red_l + 4 * R);         // [R]
    TcShared<KS, VS>* sh = reinterpret_cast<TcShared<KS, VS>*>(lim + R);
    int* kvs = reinterpret_cast<int*>(sh + 1);                // [B] kv_len
    int* cs = kvs + a.B;                                      // [B] n_clean
    int* tots = cs + a.B;                                     // [B] keys (0: not served)
    int* prefix = tots + a.B;                                 // [B*Hkv + 1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_units = a.B * a.Hkv;
    pdl_trigger();

    // ---- set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < KS; ++s) {
            mbar_init(&sh->k_full[s], 1);
            mbar_init(&sh->k_empty[s], 1);
        }
        for (int s = 0; s < VS; ++s) {
            mbar_init(&sh->v_full[s], 1);
            mbar_init(&sh->v_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh->s_full[i], 1);
            mbar_init(&sh->s_empty[i], 4 * CG);
            mbar_init(&sh->q_full[i], 1);
            mbar_init(&sh->q_empty[i], 1);
        }
        mbar_init(&sh->p_full, 4 * CG);
        mbar_init(&sh->p_empty, 1);
        mbar_init(&sh->o_full, 1);
        mbar_init(&sh->o_empty, 4 * CG);
        mbar_init(&sh->drain, 1);
        sh->abort_flag = 0;
        sh->never = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_q);
    }
    if (warp == 1) {
        tmem_alloc(&sh->tmem, kTmemCols);
        tmem_relinquish();
    }
    // Q rows past `rows` stay zero (no TMA box covers them)
    for (int i = threadIdx.x; i < (int)(2 * kQBytes / 16); i += kThreads)
        reinterpret_cast<uint4*>(sQ)[i] = make_uint4(0, 0, 0, 0);
    // everything below reads what the KV append (the preceding kernel) wrote
    pdl_wait();
    for (int b = threadIdx.x; b < a.B; b += kThreads) {
        kvs[b] = a.kv_len[b];
        cs[b] = tc_clean(a, b);
        tots[b] = tc_total_keys(a, b);
    }
    __syncthreads();
    if (warp == 0) {
        // prefix[u]: start of unit u (request u / Hkv, kv head u % Hkv) on the
        // partition axis, where a unit of nt > 0 tiles takes nt + kTcUnitCost
        int run = 0;
        for (int u0 = 0; u0 < n_units; u0 += 32) {
            const int u = u0 + lane;
            const int nt = u < n_units ? (tots[u / a.Hkv] + kTcKeys - 1) / kTcKeys : 0;
            const int w = nt > 0 ? nt + kTcUnitCost : 0;
            int incl = w;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            if (u < n_units) prefix[u] = run + incl - w;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) prefix[n_units] = run;
    }
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem;
    const int T = prefix[n_units];
    const int G = (int)gridDim.x < T ? (int)gridDim.x : T;
    const bool active = (int)blockIdx.x < G;
    const int my0 = active ? (int)((long long)T * blockIdx.x / G) : 0;
    const int my1 = active ? (int)((long long)T * (blockIdx.x + 1) / G) : 0;
    volatile int* abort_flag = &sh->abort_flag;

    // unit holding partition position pos: the largest u with prefix[u] <= pos
    auto unit_of = [&](int pos) {
        int lo = 0, hi = n_units;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (prefix[mid] <= pos) lo = mid; else hi = mid;
        }
        return lo;
    };
    auto unit_tiles = [&](int u) { return (tots[u / a.Hkv] + kTcKeys - 1) / kTcKeys; };
    // the first piece of this CTA at or after position pos (positions past a
    // unit's tiles are its epilogue share and hold no tile)
    auto piece_from = [&](int pos, TcPiece& pc) {
        while (pos < my1) {
            const int u = unit_of(pos);
            const int us = prefix[u], nt = unit_tiles(u);
            if (pos - us < nt) {
                pc.u = u;
                pc.us = us;
                pc.t0 = pos - us;
                pc.t1 = min(us + nt, my1) - us;
                pc.b = u / a.Hkv;
                pc.g = u - pc.b * a.Hkv;
                return true;
            }
            pos = prefix[u + 1];
        }
        return false;
    };
    // the piece after `cur` in this CTA's range: nothing if the range ends
    // inside cur, else the next unit with tiles from its first tile (units are
    // consecutive on the partition axis, so no search is needed)
    auto next_piece = [&](TcPiece cur, TcPiece& pc) {
        if (cur.us + cur.t1 >= my1) return false;
        for (int u = cur.u + 1; u < n_units && prefix[u] < my1; ++u) {
            const int nt = unit_tiles(u);
            if (nt > 0) {
                pc.u = u;
                pc.us = prefix[u];
                pc.t0 = 0;
                pc.t1 = min(pc.us + nt, my1) - pc.us;
                pc.b = u / a.Hkv;
                pc.g = u - pc.b * a.Hkv;
                return true;
            }
        }
        return false;
    };
    auto give_up = [&]() {
        *abort_flag = 1;
        raise_flag(a.err_flag, ISD_FLAG_WAIT_TIMEOUT);
    };

    if (warp < TcRoles<R>::kSoftWarp0) {
        // warpgroup 0: TMA producers and MMA issuer (warp 3 idles)
        if constexpr (TcRoles<R>::kRegSplit) setmaxnreg_dec<TcRoles<R>::kRegsLow>();
        if (warp == 0 || warp == TcRoles<R>::kVWarp) {
            if (active) {
                // ------------------------------------------------ TMA producers
                // Warp 0 loads Q and the K halves of the stages, the last warp the
                // V halves: each half has its own ring barriers, so a K half is
                // refilled as soon as S = K.Q^T has read it and K runs ahead of V
                // (the V half is held until P.V).  Each producer walks the tiles
                // with the whole warp: page ids come in chunks of 32 (lane i holds
                // one), the next chunk's load in flight while the current one is
                // issued, and the next piece's first chunk in flight during the
                // current piece; lane 0 waits on the ring, and the copies of a
                // half are issued one box per lane (issuing them from a single
                // thread caps the copy rate with small pages).
                const bool is_v = warp != 0;
            const int nst = is_v ? VS : KS;  // this producer's ring
                uint64_t* full = is_v ? sh->v_full : sh->k_full;
                uint64_t* empty = is_v ? sh->v_empty : sh->k_empty;
                unsigned char* ring = is_v ? sV : sK;
                const CUtensorMap* map = is_v ? &tm_v : &tm_k;
                const uint64_t pol_kv = policy_evict_first();  // each K/V byte is read once
                const uint64_t pol_q = policy_evict_last();
                const int np = kTcKeys / a.P;  // pages per tile (<= 16)
                const int tpc = 32 / np;       // tiles per chunk of page ids
                // page id of page tc0 * np + lane of the piece's request; pages
                // past the request (or bad ids) read as zeros
                auto load_ids = [&](const TcPiece& q, int tc0) {
                    const int pidx = tc0 * np + lane;
                    const int need = (tots[q.b] + a.P - 1) / a.P;
                    int id = -1;
                    if (pidx < need) {
                        id = __ldg(a.page_table + (size_t)q.b * a.max_pages + pidx);
                        if (id < 0 || id >= a.num_pages) {
                            raise_flag(a.err_flag, ISD_FLAG_PAGE_OOB);
                            id = -1;
                        }
                    }
                    return id;
                };
                int st = 0, pi = 0;
                uint32_t ph = 0, armed = 0, armed_par = 0;
                bool ok = true;
                TcPiece pc;
                bool has = piece_from(my0, pc);
                int ids_first = has ? load_ids(pc, pc.t0) : -1;
                while (ok && has) {
                    TcPiece nx;
                    const bool has_nx = next_piece(pc, nx);
                    if (!is_v) {
                        const int qb = pi & 1;
                        if (lane == 0) {
                            ok = mbar_wait_bounded(&sh->q_empty[qb], ((pi >> 1) & 1) ^ 1, abort_flag, kTcWaitNs);
                            if (!ok) {
                                give_up();
                            } else {
                                mbar_arrive_expect_tx(&sh->q_full[qb], (uint32_t)a.rows * 256u);
                                unsigned char* qd = sQ + qb * kQBytes;
                                tma_load_4d(qd, &tm_q, &sh->q_full[qb], 0, pc.g * a.grp, 0, pc.b, pol_q);
                                tma_load_4d(qd + R * 128, &tm_q, &sh->q_full[qb], 64, pc.g * a.grp, 0, pc.b, pol_q);
                            }
                        }
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                    }
                    ++pi;
                    int ids = ids_first, ids_next = load_ids(pc, pc.t0 + tpc);
                    const int ids_nx = has_nx ? load_ids(nx, nx.t0) : -1;
                    for (int t = pc.t0; t < pc.t1; ++t) {
                        const int j = (t - pc.t0) % tpc;  // tile within the chunk
                        if (j == 0 && t > pc.t0) {
                            ids = ids_next;
                            ids_next = load_ids(pc, t + tpc);
                        }
                        if (lane == 0) {
                            ok = mbar_wait_bounded(&empty[st], ph ^ 1, abort_flag, kTcWaitNs);
                            if (!ok) give_up();
                            else mbar_arrive_expect_tx(&full[st], 2u * kTcHalf);
                        }
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        unsigned char* dst = ring + st * 2 * kTcHalf;
                        // one box per lane: page lane / 2 of the tile, 64-d half lane % 2
                        // (the expect_tx above precedes them in program order)
                        for (int box0 = 0; box0 < 2 * np; box0 += 32) {
                            const int box = box0 + lane;
                            const int pg = box < 2 * np ? box >> 1 : 0, hf = box & 1;
                            const int page = __shfl_sync(0xffffffffu, ids, (j * np + pg) & 31);
                            if (box < 2 * np)
                                tma_load_4d(dst + pg * a.P * 128 + hf * kTcHalf, map, &full[st], hf * 64,
                                            pc.g, 0, page, pol_kv);
                        }
                        armed |= 1u << st;
                        armed_par = (armed_par & ~(1u << st)) | (ph << st);
                        if (++st == nst) {
                            st = 0;
                            ph ^= 1;
                        }
                    }
                    ids_first = ids_nx;
                    pc = nx;
                    has = has_nx;
                }
                // drain: every armed copy has landed before the CTA may exit
                if (lane == 0) {
                    for (int s = 0; s < nst; ++s)
                        if (armed >> s & 1)
                            mbar_wait_bounded(&full[s], armed_par >> s & 1, &sh->never, kTcWaitNs);
                    if (!is_v)
                        for (int k = pi - 1; k >= 0 && k >= pi - 2; --k)
                            mbar_wait_bounded(&sh->q_full[k & 1], (k >> 1) & 1, &sh->never, kTcWaitNs);
                }
            }
        } else if (warp == 1) {
            if (lane == 0 && active) {
                // ------------------------------------------------ MMA issuer
                constexpr uint32_t idesc_s = idesc_bf16_f32(128, R);
                constexpr uint32_t idesc_o = idesc_bf16_f32(128, R) | (1u << 15);  // A = V^T, MN-major
                const uint64_t dq0 = smem_desc_sw128(smem_u32(sQ));
                const uint64_t dk = smem_desc_sw128(smem_u32(sK));
                const uint64_t dp = smem_desc_sw128(smem_u32(sP));
                // V^T as an MN-major operand: the two 64-d blocks are kTcHalf apart
                // (leading byte offset), 8-key groups 1024 bytes apart (stride byte offset)
                const uint64_t dv = (smem_desc_sw128(smem_u32(sV)) & ~(0x3FFFull << 16)) |
                                    ((uint64_t)(kTcHalf >> 4) << 16);
                const uint32_t tm_o = tmem + 2 * R;
                // S products run ahead of the P.V products: S(t+1) is issued as
                // soon as its K half and S buffer are ready, PV(t) as soon as P(t)
                // and its V half are; the K half of a stage is released when its
                // S product completes, the V half when its P.V product does
                int s_tc = 0, s_st = 0;    // S products issued; stage of the next one
                uint32_t s_ph = 0;
                int pv_tc = 0, pv_st = 0;  // PV products issued; stage of the next one
                uint32_t pv_ph = 0;
                int pi = 0;                // pieces started
                uint32_t o_use = 0;
                uint64_t dq = dq0;
                bool ok = true;
                auto wait = [&](uint64_t* bar, uint32_t par) {
                    if (mbar_try_wait(bar, par) || mbar_wait_bounded(bar, par, abort_flag, kTcWaitNs))
                        return true;
                    give_up();
                    ok = false;
                    return false;
                };
                auto issue_s = [&]() {
                    const int buf = s_tc & 1;
                    tc_fence_after();
                    const uint32_t k_off = (uint32_t)(s_st * 2 * kTcHalf);
    #pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t ad = dk + ((k_off + (kk >> 2) * kTcHalf + (kk & 3) * 32) >> 4);
                        const uint64_t bd = dq + (((kk >> 2) * R * 128 + (kk & 3) * 32) >> 4);
                        mma_f16_ss(tmem + buf * R, ad, bd, idesc_s, kk != 0);
                    }
                    mma_commit(&sh->s_full[buf]);
                    mma_commit(&sh->k_empty[s_st]);  // the K half may be refilled once S is done
                    if (++s_st == KS) {
                        s_st = 0;
                        s_ph ^= 1;
                    }
                    ++s_tc;
                };
                auto s_inputs_ready = [&]() {
                    return mbar_test(&sh->k_full[s_st], s_ph) &&
                           mbar_test(&sh->s_empty[s_tc & 1], ((s_tc >> 1) & 1) ^ 1);
                };
                auto issue_s_blocking = [&]() {
                    if (!wait(&sh->k_full[s_st], s_ph)) return false;
                    if (!wait(&sh->s_empty[s_tc & 1], ((s_tc >> 1) & 1) ^ 1)) return false;
                    issue_s();
                    return true;
                };
                TcPiece pc;
                bool has = piece_from(my0, pc);
                while (ok && has) {
                    const int qb = pi & 1;
                    const int end_tc = s_tc + (pc.t1 - pc.t0);  // tile numbers of this piece: [s_tc, end_tc)
                    if (!wait(&sh->q_full[qb], (pi >> 1) & 1)) break;
                    ++pi;
                    dq = dq0 + ((qb * kQBytes) >> 4);
                    if (!issue_s_blocking()) break;
                    bool q_done = false, first_pv = true;
                    while (ok && pv_tc < end_tc) {
                        // wait for P(pv_tc); issue the next S meanwhile once it can go
                        const uint64_t tstart = global_ns();
                        for (uint32_t it = 0;; ++it) {
                            if (s_tc < end_tc && s_inputs_ready()) issue_s();
                            if (mbar_test(&sh->p_full, pv_tc & 1)) break;
                            if ((it & 255) == 255 && (*abort_flag || global_ns() - tstart > kTcWaitNs)) {
                                give_up();
                                ok = false;
                                break;
                            }
                        }
                        if (!ok) break;
                        if (s_tc == end_tc && !q_done) {
                            mma_commit(&sh->q_empty[qb]);  // every S product of this piece issued
                            q_done = true;
                        }
                        if (first_pv && !wait(&sh->o_empty, (o_use & 1) ^ 1)) break;
                        if (!wait(&sh->v_full[pv_st], pv_ph)) break;
                        tc_fence_after();
                        const uint32_t v_off = (uint32_t)(pv_st * 2 * kTcHalf);
    #pragma unroll
                        for (int kk = 0; kk < kTcKeys / 16; ++kk) {
                            const uint64_t ad = dv + ((v_off + kk * 2048) >> 4);
                            const uint64_t bd = dp + (((kk >> 2) * R * 128 + (kk & 3) * 32) >> 4);
                            mma_f16_ss(tm_o, ad, bd, idesc_o, (first_pv && kk == 0) ? 0u : 1u);
                        }
                        mma_commit(&sh->v_empty[pv_st]);
                        mma_commit(&sh->p_empty);
                        first_pv = false;
                        if (++pv_st == VS) {
                            pv_st = 0;
                            pv_ph ^= 1;
                        }
                        ++pv_tc;
                        // the softmax continues with S(pv_tc): issue it now if it is still missing
                        if (pv_tc < end_tc && s_tc == pv_tc && !issue_s_blocking()) break;
                    }
                    if (!ok) break;
                    if (!q_done) mma_commit(&sh->q_empty[qb]);
                    mma_commit(&sh->o_full);
                    ++o_use;
                    has = next_piece(pc, pc);
                }
                mma_commit(&sh->drain);
                mbar_wait_bounded(&sh->drain, 0, &sh->never, kTcWaitNs);
            }
        }
    } else {
        if constexpr (TcRoles<R>::kRegSplit) setmaxnreg_inc<TcRoles<R>::kRegsHigh>();
        if (active) {
            // ------------------------------------------------ softmax + epilogue
            // thread = key kl of the tile (S^T lane) and rows r0 .. r0+RC-1;
            // in the epilogue thread = output dimension d = kl of O^T
            const int q4 = warp & 3;             // TMEM lane quarter of this warp
            const int cg = (warp - TcRoles<R>::kSoftWarp0) >> 2;  // column group
            const int r0 = cg * RC;
            const int kl = q4 * 32 + lane;
            const int et = threadIdx.x - 32 * TcRoles<R>::kSoftWarp0;  // 0 .. kSoft-1
            const uint32_t tm_lane = tmem + ((uint32_t)(q4 * 32) << 16);
            // this thread's P^T column: 64-key half, swizzled 16-byte chunk, element
            const int kin = kl & 63;
            unsigned char* p_col = sP + (kl >> 6) * R * 128 + (kin & 7) * 2;
            const int p_chunk = kin >> 3;
            // one thread waits, the group follows: every thread takes the same exit
            auto group_wait = [&](uint64_t* bar, uint32_t par) -> bool {
                bool fail = false;
                if (et == 0) {
                    fail = !(mbar_try_wait(bar, par) || mbar_wait_bounded(bar, par, abort_flag, kTcWaitNs));
                    if (fail) give_up();
                }
                return !group_or<kSoft>(fail);
            };
            float m_ref[RC], l_part[RC];
            int tc = 0, kst = 0;
            uint32_t kph = 0, o_use = 0;
            bool ok = true;
            TcPiece pc;
            bool has = piece_from(my0, pc);
            while (ok && has) {
                const int u = pc.u, us = pc.us, t0 = pc.t0, t1 = pc.t1, b = pc.b, g = pc.g;
                const int kv = kvs[b], c = cs[b], total = tots[b];
                // last visible key of each row (rows are slot-major, then head in
                // the group); read after the next group barrier
                if (et < R) {
                    const int pos = et < a.rows ? tc_slot_pos(et / a.grp, kv, c, a.N) : -1;
                    lim[et] = (a.bidir && pos >= 0) ? total - 1 : min(pos, total - 1);
                }
    #pragma unroll
                for (int r = 0; r < RC; ++r) {
                    m_ref[r] = -INFINITY;
                    l_part[r] = 0.f;
                }
                for (int t = t0; t < t1; ++t) {
                    const int buf = tc & 1;
                    if (!group_wait(&sh->s_full[buf], (tc >> 1) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    __syncwarp();
                    uint32_t sr[RC];
                    tmem_load_cols<RC>(tm_lane + buf * R + r0, sr);
                    tmem_ld_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh->s_empty[buf]);
                    float s[RC];
    #pragma unroll
                    for (int r = 0; r < RC; ++r) s[r] = __uint_as_float(sr[r]) * a.scale_log2;
                    const int key = t * kTcKeys + kl;  // key index within the request
                    if (key >= kv) {
                        // block keys and the tail: the causal limit of each row
    #pragma unroll
                        for (int r = 0; r < RC; ++r)
                            if (key > lim[r0 + r]) s[r] = -INFINITY;
                    }
                    if (t * kTcKeys + kTcKeys > total) {
                        // a V row past the request's keys may hold anything: zero it,
                        // once the V half has landed, so that 0 * V stays 0 in the
                        // second product (the fence before p_full orders it)
                        if (!group_wait(&sh->v_full[kst], kph)) {
                            ok = false;
                            break;
                        }
                        if (key >= total && cg == 0) {
                            uint4* vr = reinterpret_cast<uint4*>(sV + kst * 2 * kTcHalf + kl * 128);
    #pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                vr[j] = make_uint4(0, 0, 0, 0);
                                vr[j + kTcHalf / 16] = make_uint4(0, 0, 0, 0);
                            }
                        }
                    }
                    bool need = false;
    #pragma unroll
                    for (int r = 0; r < RC; ++r) need |= s[r] > m_ref[r] + 8.f;
                    if (group_or<kSoft>(need)) {
                        // exact row maxima of this tile; move the references that it beats by > 2^8
    #pragma unroll
                        for (int r = 0; r < RC; ++r) {
                            float mx = s[r];
    #pragma unroll
                            for (int off = 16; off > 0; off >>= 1)
                                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                            if (lane == 0) red_m[(cg * 4 + q4) * RC + r] = mx;
                        }
                        group_sync<kSoft>();
                        const float* rm = red_m + cg * 4 * RC;
                        float alpha[RC];
                        bool rescale = false;
    #pragma unroll
                        for (int r = 0; r < RC; ++r) {
                            const float mx = fmaxf(fmaxf(rm[r], rm[RC + r]), fmaxf(rm[2 * RC + r], rm[3 * RC + r]));
                            alpha[r] = 1.f;
                            if (mx > m_ref[r] + 8.f) {
                                if (m_ref[r] != -INFINITY) {
                                    alpha[r] = exp2f(m_ref[r] - mx);
                                    rescale = true;
                                }
                                m_ref[r] = mx;
                            }
                            l_part[r] *= alpha[r];
                        }
                        // O^T (thread = d, column = row) is rescaled once the
                        // previous tile's product is complete
                        if (t > t0 && group_or<kSoft>(rescale)) {
                            if (!group_wait(&sh->p_empty, (tc - 1) & 1)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            __syncwarp();
                            if (rescale) {  // uniform within the warp (same rows)
                                uint32_t ov[RC];
                                tmem_load_cols<RC>(tm_lane + 2 * R + r0, ov);
                                tmem_ld_wait();
    #pragma unroll
                                for (int r = 0; r < RC; ++r)
                                    ov[r] = __float_as_uint(__uint_as_float(ov[r]) * alpha[r]);
                                tmem_store_cols<RC>(tm_lane + 2 * R + r0, ov);
                                tmem_st_wait();
                            }
                            tc_fence_before();
                        }
                    }
                    // P^T[row][key] = 2^(s - m_ref) as bf16, 128-byte-swizzled rows
                    if (tc >= 1 && !group_wait(&sh->p_empty, (tc - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    unsigned char* pcol = p_col + r0 * 128;
    #pragma unroll
                    for (int r = 0; r < RC; ++r) {
                        const float m_use = m_ref[r] == -INFINITY ? 0.f : m_ref[r];
                        const float p = exp2f(s[r] - m_use);
                        l_part[r] += p;
                        *reinterpret_cast<__nv_bfloat16*>(pcol + r * 128 + ((p_chunk ^ (r & 7)) << 4)) =
                            __float2bfloat16_rn(p);
                    }
                    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh->p_full);
                    ++tc;
                    if (++kst == VS) {
                        kst = 0;
                        kph ^= 1;
                    }
                }
                if (!ok) break;

                // ---- end of this CTA's piece of unit u: row sums, O^T, output
    #pragma unroll
                for (int r = 0; r < RC; ++r) {
                    float v = l_part[r];
    #pragma unroll
                    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                    if (lane == 0) red_l[(cg * 4 + q4) * RC + r] = v;
                }
                if (!group_wait(&sh->o_full, o_use & 1)) {  // also orders red_l
                    ok = false;
                    break;
                }
                ++o_use;
                tc_fence_after();
                __syncwarp();
                uint32_t ov[RC];
                tmem_load_cols<RC>(tm_lane + 2 * R + r0, ov);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh->o_empty);
                const float* rl = red_l + cg * 4 * RC;
                float lt[RC];
    #pragma unroll
                for (int r = 0; r < RC; ++r) lt[r] = (rl[r] + rl[RC + r]) + (rl[2 * RC + r] + rl[3 * RC + r]);
                const int d = kl;
                // output rows are staged as bf16 [rows][128] in the P buffers (free
                // until the next P write, which follows a group barrier) and then
                // written with 16-byte stores
                __nv_bfloat16* sO = reinterpret_cast<__nv_bfloat16*>(sP);
                // CTAs whose ranges meet unit u: first .. last (all non-empty)
                const long long TL = T;
                const int ue = us + unit_tiles(u);  // end of the unit's tiles on the partition axis
                const int first = (int)(((long long)(us + 1) * G + TL - 1) / TL) - 1;
                const int last = (int)(((long long)ue * G + TL - 1) / TL) - 1;
                const int npieces = last - first + 1;
                bool write_out = true;
                if (npieces == 1) {
    #pragma unroll
                    for (int r = 0; r < RC; ++r) {
                        const bool live = lim[r0 + r] >= 0 && lt[r] > 0.f;  // active row with keys
                        const float inv = live ? __frcp_rn(lt[r]) : 0.f;
                        sO[(r0 + r) * 128 + d] = __float2bfloat16_rn(__uint_as_float(ov[r]) * inv);
                    }
                } else {
                    // A unit split over CTAs first .. last: CTA first holds its
                    // first tiles and reaches them last (they end its range), the
                    // others hold later tiles at the start of their ranges.  Those
                    // leave an fp32 partial and raise its flag; CTA first merges
                    // them in CTA order into its own result (starting from its
                    // own values, exactly as if its partial were the first one
                    // read) and writes the output rows.
                    //
                    // partial slot of CTA cta for unit u: a CTA leaves a partial
                    // only for its first piece (when the unit began before its
                    // range: slot 0) and its last piece (slot 1 otherwise), so
                    // the two never share a slot
                    auto slot_of = [&](int cta) {
                        const int c0 = (int)((long long)T * cta / G);
                        return us < c0 ? 0 : 1;
                    };
                    auto part_of = [&](int cta) {
                        return a.part + ((size_t)cta * 2 + slot_of(cta)) * a.part_stride;
                    };
                    if ((int)blockIdx.x != first) {
                        float* pb = part_of(blockIdx.x);
    #pragma unroll
                        for (int r = 0; r < RC; ++r) pb[2 * R + (r0 + r) * 128 + d] = __uint_as_float(ov[r]);
                        if (kl == 0) {
    #pragma unroll
                            for (int r = 0; r < RC; ++r) {
                                pb[r0 + r] = m_ref[r];
                                pb[R + r0 + r] = lt[r];
                            }
                        }
                        __threadfence();
                        group_sync<kSoft>();
                        if (et == 0) {
                            int* f = a.part_flag + (size_t)blockIdx.x * 2 + slot_of(blockIdx.x);
                            asm volatile("st.release.gpu.global.b32 [%0], %1;\n" ::"l"(f), "r"(1) : "memory");
                        }
                        write_out = false;
                    } else {
                        float Mr[RC], Lr[RC], Or[RC];
    #pragma unroll
                        for (int r = 0; r < RC; ++r) {
                            Mr[r] = m_ref[r];
                            Lr[r] = lt[r];
                            Or[r] = __uint_as_float(ov[r]);
                        }
                        for (int cta = first + 1; cta <= last && ok; ++cta) {
                            const float* pk = part_of(cta);
                            int* f = a.part_flag + (size_t)cta * 2 + slot_of(cta);
                            // bounded wait for the partial (its CTA runs: the grid is
                            // one CTA per SM)
                            bool fail = false;
                            if (et == 0) {
                                const uint64_t t_start = global_ns();
                                for (uint32_t it = 0;; ++it) {
                                    int v;
                                    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(f) : "memory");
                                    if (v) break;
                                    if ((it & 63) == 63 && (*abort_flag || global_ns() - t_start > kTcWaitNs)) {
                                        give_up();
                                        fail = true;
                                        break;
                                    }
                                }
                            }
                            if (group_or<kSoft>(fail)) {
                                ok = false;
                                break;
                            }
                            __threadfence();
                            for (int i = et; i < R; i += kSoft) {
                                red_m[i] = __ldcg(pk + i);
                                red_l[i] = __ldcg(pk + R + i);
                            }
                            float okv[RC];
    #pragma unroll
                            for (int r = 0; r < RC; ++r) okv[r] = __ldcg(pk + 2 * R + (size_t)(r0 + r) * 128 + d);
                            group_sync<kSoft>();
    #pragma unroll
                            for (int r = 0; r < RC; ++r) {
                                const float mk = red_m[r0 + r], lk = red_l[r0 + r];
                                const float mn = fmaxf(Mr[r], mk);
                                const float mu = mn == -INFINITY ? 0.f : mn;
                                const float fa = exp2f(Mr[r] - mu), fb = exp2f(mk - mu);
                                Lr[r] = Lr[r] * fa + lk * fb;
                                Or[r] = Or[r] * fa + okv[r] * fb;
                                Mr[r] = mn;
                            }
                            group_sync<kSoft>();  // red_m / red_l are rewritten for the next partial
                            if (et == 0) *f = 0;   // consumed: clear for the next launch
                        }
                        if (!ok) break;
    #pragma unroll
                        for (int r = 0; r < RC; ++r) {
                            const bool live = lim[r0 + r] >= 0 && Lr[r] > 0.f;
                            const float inv = live ? __frcp_rn(Lr[r]) : 0.f;
                            sO[(r0 + r) * 128 + d] = __float2bfloat16_rn(Or[r] * inv);
                        }
                    }
                }
                if (write_out) {
                    group_sync<kSoft>();
                    for (int i = et; i < a.rows * 16; i += kSoft) {
                        const int r = i >> 4, ch = i & 15;
                        const int slot = r / a.grp, hh = r - slot * a.grp;
                        const uint4 v = *reinterpret_cast<const uint4*>(sO + r * 128 + ch * 8);
                        *reinterpret_cast<uint4*>(a.out + ((size_t)b * a.Q + slot) * a.Hq * 128 +
                                                  (size_t)(g * a.grp + hh) * 128 + ch * 8) = v;
                    }
                }
                // lim and the staged rows are rewritten only after the next group barrier
                group_sync<kSoft>();
                has = next_piece(pc, pc);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

bool encode_bf16_4d(CUtensorMap* m, const void* ptr, const uint64_t dims[4],
                    const uint64_t strides_bytes[3], const uint32_t box[4]) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t gd[4] = {dims[0], dims[1], dims[2], dims[3]};
    cuuint64_t gs[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
    cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), gd, gs, bx, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int R, int KS, int VS>
cudaError_t launch_tc(const TcArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                      const CUtensorMap& tq, size_t smem, cudaStream_t st, bool pdl) {
    static unsigned long long configured = 0;  // bit per device
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!(configured >> dev & 1ull)) {
        if (TcRoles<R>::kRegSplit) {
            // the register split assumes the launch allocation; a build that
            // allots fewer registers would leave the increase waiting forever
            cudaFuncAttributes fa;
            const cudaError_t ae = cudaFuncGetAttributes(&fa, attention_tc_kernel<R, KS, VS>);
            if (ae != cudaSuccess) return ae;
            if (fa.numRegs < TcRoles<R>::kLaunchRegs) {
                set_error_detail("attention: registers at launch below the warpgroup split");
                return cudaErrorInvalidConfiguration;
            }
        }
        int optin = 0;
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        const cudaError_t e = cudaFuncSetAttribute(attention_tc_kernel<R, KS, VS>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        if (e != cudaSuccess) return e;
        configured |= 1ull << dev;
    }
    return launch_kernel(pdl, attention_tc_kernel<R, KS, VS>, dim3(persistent_grid()), dim3(TcRoles<R>::kThreads),
                         smem, st, tk, tv, tq, a);
}

}  // namespace

// Tensor-core attention for D = 128, block rows per kv head <= 64 and pages
// of 8..128 tokens dividing 128.  Sets *handled = false (and launches
// nothing) when the shape or the device does not fit; the caller then uses
// the general kernel.
cudaError_t launch_attention_tc(const Plan& p, const isd_dims* d, const uint16_t* q,
                                const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_pool,
                                uint16_t* v_pool, const int32_t* page_table, const int32_t* kv_len,
                                const int32_t* n_clean, uint16_t* out, void* ws, int32_t* err_flag,
                                cudaStream_t st, int* clear_extra, int* clear_range, int clear_count,
                                bool pdl, bool bidir, bool* handled) {
    *handled = false;
    const int R = p.attn_tc_rows;
    if (R == 0) return cudaSuccess;
    int dev = 0, optin = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    // alignment slack, per-request lengths, unit offsets
    const size_t extra = 1024 + (size_t)3 * d->B * 4 + (size_t)(d->B * d->Hkv + 1) * 4;
    // the deep rings when they fit, else two stages each
    int stages = 0;
    size_t smem = 0;
    for (int s = 3; s >= 2 && !stages; --s) {
        size_t f = 0;
        if (R == 16) f = s == 3 ? tc_smem_fixed<16, kTcDeepK, kTcDeepV>() : tc_smem_fixed<16, 2, 2>();
        if (R == 32) f = s == 3 ? tc_smem_fixed<32, kTcDeepK, kTcDeepV>() : tc_smem_fixed<32, 2, 2>();
        if (R == 64) f = s == 3 ? tc_smem_fixed<64, kTcDeepK, kTcDeepV>() : tc_smem_fixed<64, 2, 2>();
        if (f + extra <= (size_t)optin) {
            stages = s;
            smem = f + extra;
        }
    }
    if (!stages || !get_encode_fn()) return cudaSuccess;
    const int Q = p.Q, P = d->page_size, Hkv = d->Hkv, Hq = d->Hq;
    CUtensorMap tk, tv, tq;
    {
        const uint64_t dims[4] = {128, (uint64_t)Hkv, (uint64_t)P, (uint64_t)d->num_pages};
        const uint64_t strides[3] = {256, (uint64_t)Hkv * 256, (uint64_t)P * Hkv * 256};
        const uint32_t box[4] = {64, 1, (uint32_t)P, 1};
        if (!encode_bf16_4d(&tk, k_pool, dims, strides, box) ||
            !encode_bf16_4d(&tv, v_pool, dims, strides, box))
            return cudaSuccess;
    }
    {
        const uint64_t dims[4] = {128, (uint64_t)Hq, (uint64_t)Q, (uint64_t)d->B};
        const uint64_t strides[3] = {256, (uint64_t)Hq * 256, (uint64_t)Q * Hq * 256};
        const uint32_t box[4] = {64, (uint32_t)p.grp, (uint32_t)Q, 1};
        if (!encode_bf16_4d(&tq, q, dims, strides, box)) return cudaSuccess;
    }
    *handled = true;
    TcArgs a;
    a.B = d->B;
    a.N = d->N;
    a.Q = Q;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.grp = p.grp;
    a.rows = p.rows;
    a.P = P;
    a.num_pages = d->num_pages;
    a.max_pages = d->max_pages_per_req;
    a.scale_log2 = d->sm_scale * 1.4426950408889634f;
    a.page_table = page_table;
    a.kv_len = kv_len;
    a.n_clean = n_clean;
    a.bidir = bidir ? 1 : 0;
    a.out = reinterpret_cast<__nv_bfloat16*>(out);
    a.part = reinterpret_cast<float*>(static_cast<char*>(ws) + p.off_attn_part);
    a.part_stride = p.attn_tc_part_stride;
    a.ticket = reinterpret_cast<int*>(static_cast<char*>(ws) + p.off_attn_ticket);
    // partial flags follow the kMaxSMs x 2 partials
    a.part_flag = reinterpret_cast<int*>(a.part + (size_t)kMaxSMs * 2 * a.part_stride);
    a.err_flag = err_flag;
    const int append_threads = (Hkv * 16 + 31) / 32 * 32;
    cudaError_t e = launch_kernel(pdl, kv_append_kernel, dim3(d->B, Q),
                                  dim3(append_threads > 1024 ? 1024 : append_threads), 0, st, a,
                                  reinterpret_cast<const __nv_bfloat16*>(k_new),
                                  reinterpret_cast<const __nv_bfloat16*>(v_new),
                                  reinterpret_cast<__nv_bfloat16*>(k_pool),
                                  reinterpret_cast<__nv_bfloat16*>(v_pool), clear_extra, clear_range,
                                  clear_count);
    if (e != cudaSuccess) return e;
    if (R == 16)
        return stages == 3 ? launch_tc<16, kTcDeepK, kTcDeepV>(a, tk, tv, tq, smem, st, pdl)
                           : launch_tc<16, 2, 2>(a, tk, tv, tq, smem, st, pdl);
    if (R == 32)
        return stages == 3 ? launch_tc<32, kTcDeepK, kTcDeepV>(a, tk, tv, tq, smem, st, pdl)
                           : launch_tc<32, 2, 2>(a, tk, tv, tq, smem, st, pdl);
    return stages == 3 ? launch_tc<64, kTcDeepK, kTcDeepV>(a, tk, tv, tq, smem, st, pdl)
                       : launch_tc<64, 2, 2>(a, tk, tv, tq, smem, st, pdl);
}

}  // namespace isd
