// LM head (a4): logits[M, V] = hidden'[M, H] . W[V, H]^T on the 5th-generation
// tensor cores, with the row statistics (a5) folded into the epilogue.
//
// Every slot's final hidden state is mapped to a vocabulary distribution
// ("I-DLM：扩散模型如何用“自省一致性”追上自回归模型质量", "ISD 核心逻辑伪代码");
// at B=32, N=4 that is M = 224 rows against a 151936 x 4096 bf16 matrix, i.e.
// 1.245 GB of weights for 279 GFLOP -- at the HBM / tensor-core ridge of a
// B200, so the kernel must stream W at full bandwidth while the tensor cores
// keep up.
//
// Design (swap-AB, persistent, warp-specialised, pairs of SMs):
//  * the vocabulary is the MMA's M dimension and the M = B*Q hidden rows its
//    N dimension (<= 256 per MMA, two N blocks up to 512), so no MMA work is
//    wasted on padding rows;
//  * the CTAs run in clusters of two that share one tcgen05.mma of M = 256
//    (cta_group::2): each CTA holds 128 vocabulary rows of W (its half of A)
//    and HALF of the hidden rows (its half of B), and its own 128 x N
//    accumulator in TMEM.  Each hidden byte therefore crosses L2 and shared
//    memory once per 256 vocabulary rows instead of once per 128, and the
//    hidden ring can be twice as deep for the same shared memory: measured
//    on B200, the depth of both rings (not the tensor or store rate) bounded
//    the single-SM version of this kernel;
//  * in each CTA warp 0 streams W tiles (64 bf16 of K per stage, 128-byte
//    swizzle, evict-first) and warp 6 the hidden half-tiles (evict-last) with
//    TMA; both CTAs' copies are counted on the leader CTA's "full" barrier;
//  * the leader's warp 1 issues the pair MMAs into double-buffered TMEM
//    accumulators and commits each stage's "empty" barrier (and each tile's
//    "accumulator full" barrier) in both CTAs at once;
//  * warps 2-5 of each CTA drain its accumulator (tcgen05.ld 32 lanes x 32
//    columns), store fp32 logits (each store instruction writes 128
//    contiguous bytes of one logits row) and keep running row statistics
//    (max, sum exp, argmax) over all the tiles the CTA finishes, reduced
//    across each warp's 32 vocabulary rows by a shuffle butterfly (no
//    shared-memory transposition); one partial per row and CTA is written at
//    the end and merged later in CTA order;
//  * the work is split "stream-K": the pair tiles' 64-column k-blocks form
//    one sequence cut into equal ranges, one per cluster, so every SM streams
//    the same number of W bytes and there is no short last wave.  A tile cut
//    by a range boundary is started by cluster c at the end of its range and
//    its remaining k-blocks are done by cluster c+1 at the start of its
//    range; c+1 leaves its fp32 accumulator in a per-CTA buffer and raises a
//    flag, and c, when it gets there, adds that buffer to its own
//    accumulator and emits the tile -- a fixed order, and in practice no
//    waiting (the buffer was written long before);
//  * every mbarrier wait is bounded (about 2 s); on time-out the CTA raises
//    ISD_FLAG_WAIT_TIMEOUT, its roles leave their loops, outstanding MMAs are
//    drained with bounded waits, and TMEM is released.  No path returns
//    early, so both CTAs of a pair reach the cluster barriers.
#include <cuda.h>

#include "common.cuh"
#include "plan.h"
#include "sm100.cuh"
#include "launch.h"
#include "tmap.h"

namespace isd {

struct LmArgs {
    int V, Mh, H;
    int BN, NB, n_acc;
    int n_pairs;                   // 256-row pair tiles
    float* part;                   // [CTA][NB*BN][128] fp32 accumulators of tile tails
    int part_stride;               // floats per CTA in part
    int* flag;                     // [CTA] 1 = part of that CTA is ready; zero at launch
    int w_stages, h_stages;
    int w_rows;                    // rows of a W box (128, or V below one tile)
    int hbox;                      // hidden rows per TMA box (BN/2 or fewer)
    uint32_t tmem_cols;
    float* logits;
    float4* stats_part;  // [Mh][gridDim.x] partial row statistics, or null
    int32_t* err_flag;
};

// per half of the epilogue warps: the four warps' row statistics of one
// 32-column group (merged into one per vocabulary tile)
constexpr int kEpiSmemBytes = 2 * 4 * 32 * 16;

// Named barriers of the eight epilogue warps: 1 and 2 for the two halves (four
// warps each, one per TMEM lane quarter), 3 for all eight; the OR form also
// tells every warp whether any of them failed.
ISD_DEVINL bool epi_all_or(bool v) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 3, 256, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}
ISD_DEVINL void epi_all_sync() { asm volatile("bar.sync 3, 256;\n" ::: "memory"); }
ISD_DEVINL void epi_half_sync(int half) {
    asm volatile("bar.sync %0, 128;\n" ::"r"(1 + half) : "memory");
}

constexpr uint64_t kWaitLimitNs = 2000000000ull;
// W producer, MMA, 8 epilogue warps, hidden producer
constexpr int kLmThreads = 352;
constexpr int kHiddenWarp = 10;
constexpr int kWStageBytes = 128 * 128;  // 128 vocabulary rows x 64 bf16

// Fast path of a bounded wait: one try_wait, then the bounded loop.
ISD_DEVINL bool lm_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    return sm100::mbar_try_wait(bar, parity) ||
           sm100::mbar_wait_bounded(bar, parity, abort, kWaitLimitNs);
}
// bounded wait with cluster-scope acquire (the barrier also counts arrivals
// from the other CTA of the pair)
ISD_DEVINL bool lm_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort) {
    if (sm100::mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = sm100::global_ns();
    for (uint32_t it = 1;; ++it) {
        if (sm100::mbar_try_wait_cluster(bar, parity)) return true;
        if ((it & 255) == 0) {
            if (*abort) return false;
            if (sm100::global_ns() - t0 > kWaitLimitNs) return false;
        }
    }
}

// Merge of two partial row statistics with one exponential (equal maxima
// keep the lower index).  Symmetric in its arguments.
ISD_DEVINL RowStat rowstat_merge1(const RowStat& a, const RowStat& b) {
    if (b.s == 0.f) return a;
    if (a.s == 0.f) return b;
    if (a.m > b.m || (a.m == b.m && a.idx < b.idx))
        return RowStat{a.m, a.s + b.s * __expf(b.m - a.m), a.idx};
    return RowStat{b.m, b.s + a.s * __expf(a.m - b.m), b.idx};
}

// Statistics of each of a lane's 32 accumulator columns over the warp's 32
// vocabulary rows, without shared memory: (1) a shuffle butterfly finds each
// column's maximum and its first row -- in the step with lane mask h every
// lane keeps half of its columns (the upper half if bit h of its lane is
// set) and compares them with its partner's copies, so after five steps lane
// l holds column l; (2) every lane fetches its columns' maxima and forms
// exp(x - max); (3) the same butterfly adds those up.  x: this lane's value
// per column; v: its vocabulary row (a multiple of 32 plus the lane); ok:
// whether v is in the vocabulary.  Lane l returns column l's statistics.
ISD_DEVINL RowStat column_stats(const uint32_t (&x)[32], int v, bool ok) {
    const int lane = threadIdx.x & 31;
    float m[16];
    int ix[16];
    {
        const bool up = lane & 16;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float keep = ok ? __uint_as_float(up ? x[j + 16] : x[j]) : -INFINITY;
            const float send = ok ? __uint_as_float(up ? x[j] : x[j + 16]) : -INFINITY;
            const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
            const bool take = recv > keep || (recv == keep && (v ^ 16) < v);
            m[j] = take ? recv : keep;
            ix[j] = take ? (v ^ 16) : v;
        }
    }
#pragma unroll
    for (int h = 8; h >= 1; h >>= 1) {
        const bool up = lane & h;
#pragma unroll
        for (int j = 0; j < h; ++j) {
            const float km = up ? m[j + h] : m[j];
            const int ki = up ? ix[j + h] : ix[j];
            const float rm = __shfl_xor_sync(0xffffffffu, up ? m[j] : m[j + h], h);
            const int ri = __shfl_xor_sync(0xffffffffu, up ? ix[j] : ix[j + h], h);
            const bool take = rm > km || (rm == km && ri < ki);
            m[j] = take ? rm : km;
            ix[j] = take ? ri : ki;
        }
    }
    float e[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float mj = __shfl_sync(0xffffffffu, m[0], j);
        e[j] = (ok && mj != -INFINITY) ? __expf(__uint_as_float(x[j]) - mj) : 0.f;
    }
    float sm[16];
    {
        const bool up = lane & 16;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            sm[j] = (up ? e[j + 16] : e[j]) + __shfl_xor_sync(0xffffffffu, up ? e[j] : e[j + 16], 16);
    }
#pragma unroll
    for (int h = 8; h >= 1; h >>= 1) {
        const bool up = lane & h;
#pragma unroll
        for (int j = 0; j < h; ++j)
            sm[j] = (up ? sm[j + h] : sm[j]) + __shfl_xor_sync(0xffffffffu, up ? sm[j] : sm[j + h], h);
    }
    return RowStat{m[0], sm[0], ix[0]};
}

// Synchronisation (per k-block `it`, W slot ws = it % w_stages, hidden slot
// hs = it % h_stages):
//   full[ws]  (leader CTA only): 2 arrivals (the leader's two producers, each
//             expecting the bytes of BOTH CTAs' copies of its operand); the
//             copies of both CTAs complete on it; the MMA thread waits on it;
//   empty[ws] (each CTA): one pair commit per k-block arrives in both CTAs.
//             The W producer reuses slot ws after it; the hidden producer
//             reuses slot hs after the commit of k-block it - h_stages, which
//             it reads from the same W-ring barrier (w_stages > h_stages keeps
//             the phases unambiguous);
//   tfull[a]  (each CTA): one pair commit per tile: accumulator a is ready;
//   tempty[a] (leader only): 16 arrivals, the 8 epilogue warps of each CTA.
template <int NB>
__global__ void __launch_bounds__(kLmThreads, 1)
lm_head_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_h,
               const __grid_constant__ LmArgs a) {
    using namespace sm100;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int half_bn = a.BN / 2;
    const int cols = NB * a.BN;
    const int h_bytes = NB * half_bn * 128;  // one hidden stage of this CTA (K = 64)
    unsigned char* wring = smem;
    unsigned char* hring = smem + (size_t)a.w_stages * kWStageBytes;
    float4* wstat = reinterpret_cast<float4*>(hring + (size_t)a.h_stages * h_bytes);  // [2][4][32]
    float4* run = wstat + 2 * 4 * 32;
    uint64_t* full = reinterpret_cast<uint64_t*>(run + cols);
    uint64_t* empty = full + a.w_stages;
    uint64_t* tfull = empty + a.w_stages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    __shared__ int never;  // a flag nothing sets: used by the final drains

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.w_stages; ++s) {
            mbar_init(&full[s], 2);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 16);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        never = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_h);
    }
    // hidden rows no copy reaches (past the matrix) read as zeros; the
    // running statistics start empty
    for (int i = threadIdx.x; i < a.h_stages * h_bytes / 16; i += kLmThreads)
        reinterpret_cast<uint4*>(hring)[i] = make_uint4(0, 0, 0, 0);
    for (int i = threadIdx.x; i < cols; i += kLmThreads)
        run[i] = make_float4(-INFINITY, 0.f, __int_as_float(0x7fffffff), 0.f);
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, a.tmem_cols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before any copy or arrival names them
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int kb = a.H / 64;  // k-blocks per tile
    // this cluster's range of the k-block sequence and the tiles it meets
    const int G2 = (int)gridDim.x >> 1;
    const int cl = (int)blockIdx.x >> 1;
    const long long U = (long long)a.n_pairs * kb;
    const long long u0 = U * cl / G2, u1 = U * (cl + 1) / G2;
    const int t_first = (int)(u0 / kb), t_last = (int)((u1 - 1) / kb);
    const int n_items = t_last - t_first + 1;
    auto item_ks = [&](int i) {  // first k-block of item i
        const long long t0 = (long long)(t_first + i) * kb;
        return (int)((u0 > t0 ? u0 : t0) - t0);
    };
    auto item_ke = [&](int i) {  // end k-block of item i
        const long long t0 = (long long)(t_first + i) * kb;
        return (int)((u1 < t0 + kb ? u1 : t0 + kb) - t0);
    };
    const int total_kb = (int)(u1 - u0);
    // bytes of one stage, both CTAs' copies together (expected by the leader)
    const uint32_t wbytes = 2u * (uint32_t)a.w_rows * 128u;
    uint32_t hbytes = 0;
    for (int nb = 0; nb < NB; ++nb)
        for (int r = 0; r < 2; ++r)
            if (nb * a.BN + r * half_bn < a.Mh) hbytes += (uint32_t)a.hbox * 128u;
    const uint32_t full_leader = mapa_shared(smem_u32(full), 0);

    auto give_up = [&]() {
        *abort_flag = 1;
        raise_flag(a.err_flag, ISD_FLAG_WAIT_TIMEOUT);
    };

    if (warp == 0 || warp == kHiddenWarp) {
        if (lane == 0) {
            // ---------------- TMA producers: warp 0 streams W from HBM through
            // the deep ring; the last warp feeds this CTA's half of the hidden tiles
            const bool is_w = (warp == 0);
            if (!is_w) pdl_wait();  // the hidden rows come from the preceding kernel
            const uint64_t pol = is_w ? policy_evict_first() : policy_evict_last();
            int ws = 0, hs = 0, item = 0;
            int k = item_ks(0), ke = item_ke(0);
            uint32_t wph = 0;
            // hidden producer: the k-block that last used its slot, as a W slot/phase
            int pws = 0;
            uint32_t pwph = 0;
            for (int it = 0; it < total_kb; ++it) {
                bool ok;
                if (is_w) {
                    ok = lm_wait(&empty[ws], wph ^ 1, abort_flag);
                } else if (it >= a.h_stages) {
                    ok = lm_wait(&empty[pws], pwph, abort_flag);
                    if (++pws == a.w_stages) { pws = 0; pwph ^= 1; }
                } else {
                    ok = true;
                }
                if (!ok) {
                    give_up();
                    break;
                }
                const int pair = t_first + item;
                const uint32_t bar = full_leader + (uint32_t)ws * 8u;
                if (is_w) {
                    if (leader) mbar_arrive_expect_tx(&full[ws], wbytes);
                    tma_load_2d_pair(wring + (size_t)ws * kWStageBytes, &tmap_w, bar, k * 64,
                                     (pair * 2 + (int)rank) * 128, pol);
                } else {
                    if (leader) mbar_arrive_expect_tx(&full[ws], hbytes);
                    unsigned char* sb = hring + (size_t)hs * h_bytes;
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) {
                        const int row = nb * a.BN + (int)rank * half_bn;
                        if (row < a.Mh)
                            tma_load_2d_pair(sb + nb * half_bn * 128, &tmap_h, bar, k * 64, row, pol);
                    }
                }
                if (++ws == a.w_stages) { ws = 0; wph ^= 1; }
                if (++hs == a.h_stages) hs = 0;
                if (++k == ke) {
                    ++item;
                    if (item < n_items) {
                        k = item_ks(item);
                        ke = item_ke(item);
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------- MMA issuer (leader CTA): one pair MMA computes
            // both CTAs' 128 vocabulary rows against all BN hidden rows
            const uint32_t idesc = idesc_bf16_f32(256, a.BN);
            const uint64_t adesc0 = smem_desc_sw128(smem_u32(wring));
            const uint64_t bdesc0 = smem_desc_sw128(smem_u32(hring));
            const uint64_t astep = kWStageBytes >> 4, bstep = (uint64_t)(h_bytes >> 4);
            const uint64_t nbstep = (uint64_t)((half_bn * 128) >> 4);
            int ws = 0, hs = 0;
            uint32_t wph = 0;
            bool ok = true;
            for (int lt = 0; ok && lt < n_items; ++lt) {
                const int acc = lt % a.n_acc;
                const uint32_t use = (uint32_t)(lt / a.n_acc);
                if (!lm_wait_cluster(&tempty[acc], (use & 1) ^ 1, abort_flag)) {
                    give_up();
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(acc * cols);
                const int len = item_ke(lt) - item_ks(lt);
                for (int j = 0; j < len; ++j) {
                    if (!lm_wait(&full[ws], wph, abort_flag)) {
                        give_up();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = adesc0 + (uint64_t)ws * astep;
                    const uint64_t bd = bdesc0 + (uint64_t)hs * bstep;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb)
                            mma_f16_ss_pair(d0 + nb * a.BN, ad + 2 * k, bd + nb * nbstep + 2 * k,
                                            idesc, (j | k) != 0);
                    }
                    mma_commit_pair(&empty[ws], 0x3);
                    if (++ws == a.w_stages) { ws = 0; wph ^= 1; }
                    if (++hs == a.h_stages) hs = 0;
                }
                if (ok) mma_commit_pair(&tfull[acc], 0x3);
            }
            // all issued MMAs complete (in both CTAs) before TMEM is released
            mma_commit_pair(drain, 0x3);
        }
        if (lane == 0) mbar_wait_bounded(drain, 0, &never, kWaitLimitNs);
        __syncwarp();
    } else {
        // ---------------- epilogue: warps 2..9; warp w reads TMEM lane quarter
        // w % 4, and the two halves (warps 2-5, 6-9) take alternate 32-column groups
        const int quarter = warp & 3;
        const int ehalf = (warp - 2) >> 2;
        pdl_wait();  // logits, statistics and counters are shared with earlier kernels
        const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0);
        const int vl = quarter * 32 + lane;   // this lane's row of the 128-row tile
        float* mine = a.part + (size_t)blockIdx.x * a.part_stride;
        float4* ws4 = wstat + ehalf * 4 * 32;
        // the CTA whose buffer completes this CTA's last tile: same rank, next cluster
        const int partner = (int)blockIdx.x + 2;
        const int gpb = (a.BN + 31) / 32;     // 32-column groups per N block
        for (int lt = 0; lt < n_items; ++lt) {
            const int half = (t_first + lt) * 2 + (int)rank;  // this CTA's 128-row tile
            const bool tail = item_ks(lt) > 0;              // started by the previous cluster
            const bool head = item_ke(lt) < kb;             // finished with the next cluster's part
            const int acc = lt % a.n_acc;
            const uint32_t use = (uint32_t)(lt / a.n_acc);
            int ok = 1;
            if (lane == 0) {
                ok = lm_wait(&tfull[acc], use & 1, abort_flag);
                if (!ok) give_up();
            }
            // the eight epilogue warps meet at named barriers: they leave together
            if (epi_all_or(!ok)) break;
            tc_fence_after();
            const int v = half * 128 + vl;
            const bool v_ok = v < a.V;
            const uint32_t taddr =
                tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * cols);
            // bn is a multiple of 16: the last column group may be one
            // 16-column load, so no load reaches past the allocated columns
            auto load_cols = [&](uint32_t taddr_c, int ncols, uint32_t (&r)[32]) {
                if (ncols >= 32)
                    tmem_ld_32x32b_x32(taddr_c, r);
                else
                    tmem_ld_32x32b_x16(taddr_c, r);
                tmem_ld_wait();
            };
            // this warp is done with the accumulator: tell the leader's MMA thread
            auto release_acc = [&]() {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (leader) mbar_arrive(&tempty[acc]);
                    else mbar_arrive_remote(tempty_leader + (uint32_t)acc * 8u);
                }
            };
            if (tail) {
                // the later k-blocks of a tile this CTA does not finish: leave
                // them (fp32, column-major, lanes = vocabulary rows) for the
                // previous cluster and raise this CTA's flag
                for (int g = ehalf; g < NB * gpb; g += 2) {
                    const int nb = g / gpb, j0 = (g % gpb) * 32;
                    uint32_t r[32];
                    load_cols(taddr + nb * a.BN + j0, a.BN - j0, r);
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if (j0 + k < a.BN)
                            mine[(size_t)(nb * a.BN + j0 + k) * 128 + vl] = __uint_as_float(r[k]);
                }
                release_acc();
                __threadfence();
                epi_all_sync();
                if (warp == 2 && lane == 0) atomicExch(&a.flag[blockIdx.x], 1);
                continue;
            }
            const float* other = nullptr;
            if (head) {
                // the rest of this tile is in the partner's buffer (written at
                // the start of its range); bounded wait for its flag
                int ready = 1;
                if (warp == 2 && lane == 0) {
                    const uint64_t t0 = global_ns();
                    for (uint32_t it = 0;; ++it) {
                        int f;
                        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(f) : "l"(a.flag + partner) : "memory");
                        if (f) break;
                        if ((it & 63) == 63 && (*abort_flag || global_ns() - t0 > kWaitLimitNs)) {
                            ready = 0;
                            give_up();
                            break;
                        }
                    }
                }
                if (epi_all_or(!ready)) {
                    release_acc();
                    break;
                }
                other = a.part + (size_t)partner * a.part_stride;
            }
            float4* part = a.stats_part;
            for (int g = ehalf; g < NB * gpb; g += 2) {
                const int nb = g / gpb, j0 = (g % gpb) * 32;
                uint32_t r[32];
                load_cols(taddr + nb * a.BN + j0, a.BN - j0, r);
                if (other) {
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if (j0 + k < a.BN)
                            r[k] = __float_as_uint(__uint_as_float(r[k]) +
                                                   __ldcg(other + (size_t)(nb * a.BN + j0 + k) * 128 + vl));
                }
                const int mbase = nb * a.BN + j0;  // hidden row of column j0
                if (v_ok) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const int m = mbase + k;
                        if (j0 + k < a.BN && m < a.Mh) a.logits[(size_t)m * a.V + v] = __uint_as_float(r[k]);
                    }
                }
                if (!part) continue;
                // row statistics of this warp's 32 vocabulary rows, then the
                // four warps' merged in vocabulary order into the running ones
                const RowStat st = column_stats(r, v, v_ok);
                ws4[quarter * 32 + lane] = make_float4(st.m, st.s, __int_as_float(st.idx), 0.f);
                epi_half_sync(ehalf);
                if (quarter == 0) {
                    RowStat t = rowstat_empty();
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 e = ws4[q * 32 + lane];
                        t = rowstat_merge1(t, RowStat{e.x, e.y, __float_as_int(e.z)});
                    }
                    if (j0 + lane < a.BN && mbase + lane < a.Mh) {
                        const float4 o = run[mbase + lane];
                        const RowStat mrg = rowstat_merge1(RowStat{o.x, o.y, __float_as_int(o.z)}, t);
                        run[mbase + lane] = make_float4(mrg.m, mrg.s, __int_as_float(mrg.idx), 0.f);
                    }
                }
                epi_half_sync(ehalf);
            }
            release_acc();
            if (head) {
                epi_all_sync();  // every warp has read the partner's buffer
                if (warp == 2 && lane == 0) a.flag[partner] = 0;
            }
        }
        // the running statistics: one partial per row and CTA
        epi_all_sync();
        if (a.stats_part && warp == 2) {
            for (int c0 = 0; c0 < cols; c0 += 32) {
                const int col = c0 + lane;  // running column == hidden row
                if (col < cols && col < a.Mh)
                    a.stats_part[(size_t)col * gridDim.x + blockIdx.x] = run[col];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no copy, arrival or commit names the other CTA after this
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, a.tmem_cols);
    }
}

// Row statistics from the LM head's partials: one warp per row merges that
// row's n_parts partials with warp_merge_partials (the routine and order the
// accept kernel uses when it merges them inside a whole step).
__global__ void __launch_bounds__(256)
lm_stats_merge_kernel(const float4* __restrict__ part, int n_parts, int rows,
                      isd_row_stat* __restrict__ out) {
    pdl_trigger();
    pdl_wait();
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const RowStat st = warp_merge_partials(part + (size_t)row * n_parts, n_parts);
    if ((threadIdx.x & 31) == 0) out[row] = isd_row_stat{st.m, st.s, st.idx, 0};
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// 2-D bf16 [rows, cols] row-major tensor, box = 64 columns x box_rows rows, 128B swizzle.
static bool encode_bf16_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols,
                           uint32_t box_rows) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

struct LmShape {
    int BN, NB, n_acc, w_stages, h_stages;
    uint32_t tmem_cols;
    size_t smem;
};

static bool lm_head_shape(int Mh, int smem_limit, LmShape* s) {
    if (Mh < 1 || Mh > 512) return false;
    s->NB = Mh <= 256 ? 1 : 2;
    s->BN = lm_cols(Mh) / s->NB;
    const int cols = s->NB * s->BN;
    s->n_acc = (2 * cols <= 512) ? 2 : 1;
    const int need = s->n_acc * cols;
    uint32_t alloc = 32;
    while ((int)alloc < need) alloc <<= 1;
    s->tmem_cols = alloc;
    const int h_bytes = s->NB * (s->BN / 2) * 128;
    // slack, barriers, the epilogue warps' statistics, running statistics
    const int fixed = 1024 + 512 + kEpiSmemBytes + cols * 16;
    const int budget = smem_limit - fixed;
    // hidden tiles come from L2, but under load their latency is long: up to
    // 4 stages while the W ring keeps at least twice as many, else the
    // deepest hidden ring that leaves W more stages than hidden
    s->h_stages = 0;
    s->w_stages = 0;
    for (int pass = 0; pass < 2 && !s->h_stages; ++pass) {
        for (int h = 4; h >= 2; --h) {
            int w = (budget - h * h_bytes) / kWStageBytes;
            if (w > 16) w = 16;
            if (pass == 0 ? w >= 2 * h : w > h) {
                s->h_stages = h;
                s->w_stages = w;
                break;
            }
        }
    }
    if (!s->h_stages) return false;
    s->smem = (size_t)s->w_stages * kWStageBytes + (size_t)s->h_stages * h_bytes + fixed;
    return true;
}

void set_error_detail(const char* msg);

// Grid of the LM head for these shapes on the current device: an even number
// of CTAs (clusters of two), at most two per pair tile.
static int lm_grid(int V) {
    const int n_pairs = ((V + 127) / 128 + 1) / 2;
    int grid = persistent_grid() & ~1;
    if (grid < 2) grid = 2;
    if (grid > 2 * n_pairs) grid = 2 * n_pairs;
    return grid;
}

// Row-statistics partials per row that launch_lm_head writes: one per CTA.
int lm_head_stat_parts(int Mh, int H, int V) {
    (void)Mh;
    (void)H;
    return lm_grid(V);
}

// pdl: launched as part of the whole step (programmatic dependent launch);
// counters_cleared: an earlier kernel of the step already cleared the flags
// of the tile-tail buffers in tail_ws.
cudaError_t launch_lm_head(const uint16_t* hidden, const uint16_t* W, int Mh, int H, int V,
                           float* logits, float4* stats_part, void* tail_ws, int32_t* err_flag,
                           cudaStream_t st, bool pdl, bool counters_cleared) {
    // dynamic shared memory available to this kernel on the current device
    static int smem_limit_dev[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!smem_limit_dev[dev]) {
        int optin = 0;
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaFuncAttributes fa1, fa2;
        if (cudaFuncGetAttributes(&fa1, lm_head_kernel<1>) != cudaSuccess ||
            cudaFuncGetAttributes(&fa2, lm_head_kernel<2>) != cudaSuccess) {
            set_error_detail("lm_head: kernel attributes unavailable");
            return cudaErrorInvalidValue;
        }
        const size_t stat = fa1.sharedSizeBytes > fa2.sharedSizeBytes ? fa1.sharedSizeBytes
                                                                       : fa2.sharedSizeBytes;
        const int limit = optin - (int)stat;
        if (cudaFuncSetAttribute(lm_head_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 limit) != cudaSuccess ||
            cudaFuncSetAttribute(lm_head_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 limit) != cudaSuccess) {
            set_error_detail("lm_head: shared-memory attribute rejected");
            return cudaErrorInvalidValue;
        }
        smem_limit_dev[dev] = limit;
    }
    LmShape sh;
    if (!lm_head_shape(Mh, smem_limit_dev[dev], &sh)) {
        set_error_detail("lm_head: no tile shape for these rows");
        return cudaErrorInvalidValue;
    }
    if (!get_encode_fn()) {
        set_error_detail("lm_head: cuTensorMapEncodeTiled entry point not found");
        return cudaErrorInvalidValue;
    }
    const int grid = lm_grid(V);
    if (grid > kMaxStatParts || grid > kMaxSMs || !tail_ws) {
        set_error_detail("lm_head: grid beyond the workspace layout");
        return cudaErrorInvalidValue;
    }
    LmArgs a;
    a.V = V;
    a.Mh = Mh;
    a.H = H;
    a.BN = sh.BN;
    a.NB = sh.NB;
    a.n_acc = sh.n_acc;
    a.w_stages = sh.w_stages;
    a.h_stages = sh.h_stages;
    a.n_pairs = ((V + 127) / 128 + 1) / 2;
    a.tmem_cols = sh.tmem_cols;
    a.logits = logits;
    a.stats_part = stats_part;
    a.err_flag = err_flag;
    a.w_rows = V < 128 ? V : 128;
    a.hbox = sh.BN / 2 < Mh ? sh.BN / 2 : Mh;
    a.part_stride = lm_part_floats(Mh);
    a.part = static_cast<float*>(tail_ws);
    a.flag = reinterpret_cast<int*>(static_cast<char*>(tail_ws) +
                                    (size_t)kMaxSMs * lm_part_floats(Mh) * 4);
    CUtensorMap tw, th;
    if (!encode_bf16_2d(&tw, W, (uint64_t)V, (uint64_t)H, (uint32_t)a.w_rows)) {
        set_error_detail("lm_head: tensor map of W rejected");
        return cudaErrorInvalidValue;
    }
    if (!encode_bf16_2d(&th, hidden, (uint64_t)Mh, (uint64_t)H, (uint32_t)a.hbox)) {
        set_error_detail("lm_head: tensor map of hidden rejected");
        return cudaErrorInvalidValue;
    }
    if (!counters_cleared) {
        const cudaError_t me = cudaMemsetAsync(a.flag, 0, (size_t)grid * 4, st);
        if (me != cudaSuccess) {
            set_error_detail("lm_head: clearing the tile-tail flags");
            return me;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kLmThreads);
    cfg.dynamicSmemBytes = sh.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    cudaError_t e = sh.NB == 1 ? cudaLaunchKernelEx(&cfg, lm_head_kernel<1>, tw, th, a)
                               : cudaLaunchKernelEx(&cfg, lm_head_kernel<2>, tw, th, a);
    if (e != cudaSuccess) set_error_detail("lm_head: launch failed");
    return e;
}

cudaError_t launch_lm_stats_merge(const float4* part, int n_parts, int rows, isd_row_stat* out,
                                  cudaStream_t st, bool pdl) {
    return launch_kernel(pdl, lm_stats_merge_kernel, dim3((rows + 7) / 8), dim3(256), 0, st, part,
                         n_parts, rows, out);
}

}  // namespace isd
