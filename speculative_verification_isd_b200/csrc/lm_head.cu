// LM head (a4): logits[M, V] = hidden'[M, H] . W[V, H]^T on the 5th-generation
// tensor cores.
//
// Every slot's final hidden state is mapped to a vocabulary distribution
// ("I-DLM：扩散模型如何用“自省一致性”追上自回归模型质量", "ISD 核心逻辑伪代码");
// at B=32, N=4 that is M = 224 rows against a 151936 x 4096 bf16 matrix, i.e.
// 1.245 GB of weights for 279 GFLOP -- at the HBM / tensor-core ridge of a
// B200, so the kernel must stream W at full bandwidth while the tensor cores
// keep up.
//
// Design (swap-AB, persistent, warp-specialised, one CTA per SM):
//  * the vocabulary is the MMA's M dimension (128-row tiles of W are operand
//    A) and the M = B*Q hidden rows are its N dimension (<= 256 per MMA, two
//    N blocks up to 512), so no MMA work is wasted on padding rows;
//  * warp 0 lane 0 streams W and hidden tiles (64 bf16 of K per stage, 128-byte
//    swizzle) into a multi-stage shared-memory ring with TMA; W is marked
//    evict-first in L2, the small hidden matrix evict-last;
//  * warp 1 lane 0 issues tcgen05.mma (M=128, N=BN, K=16) into a TMEM
//    accumulator, double-buffered when it fits in 512 columns, and releases
//    ring stages with tcgen05.commit;
//  * warps 2-5 drain the accumulator (tcgen05.ld 32 lanes x 32 columns) and
//    store fp32 logits: lanes are consecutive vocabulary entries, so each
//    store instruction writes 128 contiguous bytes of one logits row;
//  * the vocabulary tiles are dealt round-robin in whole waves of gridDim.x;
//    the L < gridDim.x tiles left over are split along N (the hidden rows)
//    into chunks of 16-row multiples, so the last wave is short instead of
//    one tile long; the chunk CTAs read their shared W tile in the same order
//    with an L2-keep hint, so it crosses HBM about once.  When CTAs are still
//    idle, each chunk is also split into K slices: every slice writes an fp32
//    partial, and the last slice to finish sums them in K order before the
//    usual epilogue (logits and fused row statistics), so the result does not
//    depend on timing;
//  * every mbarrier wait is bounded (about 2 s); on time-out the CTA raises
//    ISD_FLAG_WAIT_TIMEOUT, every role leaves its loop, outstanding TMA loads
//    and MMAs are drained with bounded waits, and TMEM is released.
#include <cuda.h>

#include "common.cuh"
#include "plan.h"
#include "sm100.cuh"
#include "launch.h"
#include "tmap.h"

namespace isd {

struct LmArgs {
    int V, Mh, H;
    int BN, n_acc, n_tiles;
    int n_full;                    // tiles dealt in whole waves (a multiple of gridDim.x)
    int tail_split;                // chunks per left-over tile (1: left-over tiles are whole)
    int tail_bn;                   // hidden rows per chunk (multiple of 16)
    int tail_ksplit;               // K slices per chunk (1: a chunk runs the whole K loop)
    float* tail_part;              // [chunk CTA][tail_bn][128] fp32 K-slice partials
    int* tail_ticket;              // [left-over tiles * tail_split], zero at launch
    int w_stages, h_stages;        // depth of the W ring and of the hidden ring (w > h)
    int w_rows, h_rows0, h_rows1;  // TMA box heights (never taller than the tensor)
    uint32_t tmem_cols;
    float* logits;
    float4* stats_part;  // [Mh][n_tiles] partial row statistics, or null
    int32_t* err_flag;
};

constexpr int kEpiPitch = 33;  // floats per row of an epilogue transposition buffer
// four transposition buffers, then the four warps' row statistics of one
// 32-column group (merged into one partial per vocabulary tile)
constexpr int kEpiSmemBytes = 4 * 32 * kEpiPitch * 4 + 4 * 32 * 16;

// named barrier 1 over the four epilogue warps; OR of a predicate
ISD_DEVINL bool epi_or(bool v) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, 128, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}
ISD_DEVINL void epi_sync() { asm volatile("bar.sync 1, 128;\n" ::: "memory"); }

constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kLmThreads = 224;  // W producer, MMA, 4 epilogue warps, hidden producer
constexpr int kWStageBytes = 128 * 128;  // 128 vocabulary rows x 64 bf16

// Fast path of a bounded wait: one try_wait, then the bounded loop.
ISD_DEVINL bool lm_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    return sm100::mbar_try_wait(bar, parity) ||
           sm100::mbar_wait_bounded(bar, parity, abort, kWaitLimitNs);
}

// Synchronisation (per k-block `it`, W slot ws = it % w_stages, hidden slot
// hs = it % h_stages):
//   full[ws]  : 2 arrivals (both producers, with their TMA byte counts); the
//               MMA thread waits on it alone;
//   empty[ws] : one tcgen05.commit per k-block.  The W producer reuses slot ws
//               after it; the hidden producer reuses slot hs after the commit
//               of k-block it - h_stages, which it reads from the same W-ring
//               barrier (w_stages > h_stages keeps the phases unambiguous).
// The MMA thread's loop is kept to one wait, the MMAs and one commit: the
// tensor pipe queues only a couple of MMAs, so any extra work there would
// become a bubble.
template <int NB>
__global__ void __launch_bounds__(kLmThreads, 1)
lm_head_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_h0,
               const __grid_constant__ CUtensorMap tmap_h1, const __grid_constant__ CUtensorMap tmap_ht,
               LmArgs a) {
    using namespace sm100;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int h_bytes = NB * a.BN * 128;  // one hidden stage (K = 64)
    unsigned char* wring = smem;
    unsigned char* hring = smem + (size_t)a.w_stages * kWStageBytes;
    float* epi_buf = reinterpret_cast<float*>(hring + (size_t)a.h_stages * h_bytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(epi_buf) +
                                                 kEpiSmemBytes);
    uint64_t* empty = full + a.w_stages;
    uint64_t* tfull = empty + a.w_stages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    __shared__ int never;  // a flag nothing sets: used by the final drains

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.w_stages; ++s) {
            mbar_init(&full[s], 2);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        never = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_h0);
        if (NB > 1) prefetch_tmap(&tmap_h1);
        if (a.tail_split > 1) prefetch_tmap(&tmap_ht);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, a.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int kblocks = a.H / 64;
    // Each CTA starts its K loop at a different block so that the 148 CTAs
    // read different hidden slices at any moment.
    const int kb0 = (int)(blockIdx.x % (unsigned)kblocks);
    // Work items of this CTA: its tiles of the whole waves, then at most one
    // left-over tile (whole) or one chunk of a left-over tile.
    const int G = (int)gridDim.x;
    const int n_wave = a.n_full / G;
    const int n_left = a.n_tiles - a.n_full;
    const int S = a.tail_split, KS = a.tail_ksplit;
    const bool has_extra = (int)blockIdx.x < n_left * S * KS;
    const int grp = (int)blockIdx.x / KS;     // left-over tile * S + row chunk of this CTA
    const int kslice = (int)blockIdx.x % KS;  // its K slice of that chunk
    const int kb_lo = kslice * kblocks / KS, kb_hi = (kslice + 1) * kblocks / KS;
    const int n_my_tiles = n_wave + (has_extra ? 1 : 0);
    auto item_tile = [&](int i) {
        return i < n_wave ? (int)blockIdx.x + i * G : a.n_full + grp / S;
    };
    auto item_is_chunk = [&](int i) { return i >= n_wave && S > 1; };
    auto item_len = [&](int i) { return item_is_chunk(i) ? kb_hi - kb_lo : kblocks; };
    const int total_kb = n_wave * kblocks + (has_extra ? item_len(n_wave) : 0);
    const int chunk_row0 = (grp % S) * a.tail_bn;  // first hidden row of this CTA's chunk

    auto give_up = [&]() {
        *abort_flag = 1;
        raise_flag(a.err_flag, ISD_FLAG_WAIT_TIMEOUT);
    };

    if (warp == 0 || warp == 6) {
        if (lane == 0) {
            // ---------------- TMA producers: warp 0 streams W from HBM through
            // the deep ring; warp 6 feeds the L2-resident hidden tiles
            const bool is_w = (warp == 0);
            // under programmatic dependent launch W (which no earlier kernel
            // of the step writes) streams at once; the hidden rows come from
            // the preceding kernel and wait for it
            if (!is_w) pdl_wait();
            const uint64_t pol = is_w ? policy_evict_first() : policy_evict_last();
            const uint64_t pol_keep = policy_evict_last();
            int ws = 0, hs = 0, kb = kb0, item = 0, jt = 0;
            int tile = item_tile(0);
            bool chunk = item_is_chunk(0);
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
                // a chunk walks its K slice in order, like the other chunks of its tile
                const int kbi = chunk ? kb_lo + jt : kb;
                if (is_w) {
                    mbar_arrive_expect_tx(&full[ws], (uint32_t)a.w_rows * 128u);
                    tma_load_2d(wring + (size_t)ws * kWStageBytes, &tmap_w, &full[ws], kbi * 64,
                                tile * 128, chunk ? pol_keep : pol);
                } else if (chunk) {
                    mbar_arrive_expect_tx(&full[ws], (uint32_t)a.tail_bn * 128u);
                    tma_load_2d(hring + (size_t)hs * h_bytes, &tmap_ht, &full[ws], kbi * 64, chunk_row0, pol);
                } else {
                    mbar_arrive_expect_tx(&full[ws], (uint32_t)(a.h_rows0 + a.h_rows1) * 128u);
                    unsigned char* sb = hring + (size_t)hs * h_bytes;
                    tma_load_2d(sb, &tmap_h0, &full[ws], kbi * 64, 0, pol);
                    if (NB > 1) tma_load_2d(sb + a.BN * 128, &tmap_h1, &full[ws], kbi * 64, a.BN, pol);
                }
                if (++ws == a.w_stages) { ws = 0; wph ^= 1; }
                if (++hs == a.h_stages) hs = 0;
                if (++kb == kblocks) kb = 0;
                if (++jt == item_len(item)) {
                    jt = 0;
                    ++item;
                    tile = item_tile(item);
                    chunk = item_is_chunk(item);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            const uint32_t idesc_full = idesc_bf16_f32(128, a.BN);
            const uint32_t idesc_chunk = idesc_bf16_f32(128, a.tail_bn);
            const uint64_t adesc0 = smem_desc_sw128(smem_u32(wring));
            const uint64_t bdesc0 = smem_desc_sw128(smem_u32(hring));
            const uint64_t astep = kWStageBytes >> 4, bstep = (uint64_t)(h_bytes >> 4);
            int ws = 0, hs = 0;
            uint32_t wph = 0;
            bool ok = true;
            for (int lt = 0; ok && lt < n_my_tiles; ++lt) {
                const int acc = lt % a.n_acc;
                const uint32_t use = (uint32_t)(lt / a.n_acc);
                if (!lm_wait(&tempty[acc], (use & 1) ^ 1, abort_flag)) {
                    give_up();
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(acc * NB * a.BN);
                const bool chunk = item_is_chunk(lt);
                const uint32_t idesc = chunk ? idesc_chunk : idesc_full;
                const int nbs = chunk ? 1 : NB;
                const int len = item_len(lt);
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
                            if (nb < nbs)
                                mma_f16_ss(d0 + nb * a.BN, ad + 2 * k,
                                           bd + (uint64_t)(nb * a.BN * 8) + 2 * k, idesc, (j | k) != 0);
                    }
                    mma_commit(&empty[ws]);
                    if (++ws == a.w_stages) { ws = 0; wph ^= 1; }
                    if (++hs == a.h_stages) hs = 0;
                }
                if (ok) mma_commit(&tfull[acc]);
            }
            // all issued MMAs complete before TMEM is released
            mma_commit(drain);
            mbar_wait_bounded(drain, 0, &never, kWaitLimitNs);
        }
    } else {
        // ---------------- epilogue: warps 2..5 cover TMEM lane quarters 2,3,0,1
        const int quarter = warp & 3;
        pdl_wait();  // logits, statistics and counters are shared with earlier kernels
        for (int lt = 0; lt < n_my_tiles; ++lt) {
            const int tile = item_tile(lt);
            const bool chunk = item_is_chunk(lt);
            const int bn = chunk ? a.tail_bn : a.BN;    // accumulator columns of this item
            const int nbs = chunk ? 1 : NB;
            const int row0 = chunk ? chunk_row0 : 0;    // hidden row of column 0
            const int acc = lt % a.n_acc;
            const uint32_t use = (uint32_t)(lt / a.n_acc);
            int ok = 1;
            if (lane == 0) {
                ok = lm_wait(&tfull[acc], use & 1, abort_flag);
                if (!ok) give_up();
            }
            // the four epilogue warps meet at named barriers: they leave together
            if (epi_or(!ok)) break;
            tc_fence_after();
            const int v = tile * 128 + quarter * 32 + lane;
            const bool v_ok = v < a.V;
            const int nvalid = a.V - (tile * 128 + quarter * 32);  // valid vocab rows of this warp
            const uint32_t taddr =
                tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * NB * a.BN);
            float* tb = epi_buf + quarter * 32 * kEpiPitch;
            float4* part = a.stats_part;
            float4* wstat = reinterpret_cast<float4*>(epi_buf + 4 * 32 * kEpiPitch);  // [4][32]
            // logits and merged row statistics of accumulator columns j0..j0+31
            // (hidden rows mbase..), one value per column in r[]
            auto emit = [&](const uint32_t (&r)[32], int j0, int mbase) {
                if (v_ok) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const int m = mbase + k;
                        if (j0 + k < bn && m < a.Mh) a.logits[(size_t)m * a.V + v] = __uint_as_float(r[k]);
                    }
                }
                if (!part) return;
                // Row statistics of this warp's 32 vocabulary entries: transpose
                // through shared memory so that lane k holds logits row mbase + k,
                // then max / sum-exp / argmax (first index among equal maxima).
#pragma unroll
                for (int k = 0; k < 32; ++k) tb[lane * kEpiPitch + k] = __uint_as_float(r[k]);
                __syncwarp();
                float x[32];
                float mx = -INFINITY;
                int arg = 0;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x[i] = tb[i * kEpiPitch + lane];
                    if (i < nvalid && x[i] > mx) {
                        mx = x[i];
                        arg = i;
                    }
                }
                float se = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i < nvalid) se += __expf(x[i] - mx);
                // the four warps' statistics of row m merged in vocabulary
                // order into one partial per tile
                wstat[quarter * 32 + lane] =
                    make_float4(mx, se, __int_as_float(tile * 128 + quarter * 32 + arg), 0.f);
                epi_sync();
                if (quarter == 0) {
                    RowStat st = rowstat_empty();
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 e = wstat[q * 32 + lane];
                        st = rowstat_merge(st, RowStat{e.x, e.y, __float_as_int(e.z)});
                    }
                    const int m = mbase + lane;
                    if (j0 + lane < bn && m < a.Mh)
                        part[(size_t)m * a.n_tiles + tile] = make_float4(st.m, st.s, __int_as_float(st.idx), 0.f);
                }
                epi_sync();
            };
            // bn is a multiple of 16: the last column group may be one
            // 16-column load, so no load reaches past the allocated columns
            auto load_cols = [&](uint32_t taddr_c, int ncols, uint32_t (&r)[32]) {
                if (ncols >= 32)
                    tmem_ld_32x32b_x32(taddr_c, r);
                else
                    tmem_ld_32x32b_x16(taddr_c, r);
                tmem_ld_wait();
            };
            if (!(chunk && KS > 1)) {
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    if (nb >= nbs) break;
                    for (int j0 = 0; j0 < bn; j0 += 32) {
                        uint32_t r[32];
                        load_cols(taddr + nb * a.BN + j0, bn - j0, r);
                        emit(r, j0, row0 + nb * a.BN + j0);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
            } else {
                // One K slice of a row chunk: the fp32 partial goes to this CTA's
                // slot (column-major, lanes = vocabulary rows); the last slice to
                // finish sums the slices in K order and emits the chunk.
                const int vl = quarter * 32 + lane;
                float* mine = a.tail_part + (size_t)blockIdx.x * bn * 128;
                for (int j0 = 0; j0 < bn; j0 += 32) {
                    uint32_t r[32];
                    load_cols(taddr + j0, bn - j0, r);
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if (j0 + k < bn) mine[(size_t)(j0 + k) * 128 + vl] = __uint_as_float(r[k]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
                __threadfence();
                epi_sync();
                bool last = false;
                if (quarter == 0 && lane == 0) last = atomicAdd(&a.tail_ticket[grp], 1) == KS - 1;
                if (epi_or(last)) {
                    __threadfence();
                    const float* slices = a.tail_part + (size_t)grp * KS * bn * 128;
                    for (int j0 = 0; j0 < bn; j0 += 32) {
                        uint32_t r[32];
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            float acc_v = 0.f;
                            if (j0 + k < bn)
                                for (int q = 0; q < KS; ++q)
                                    acc_v += __ldcg(slices + ((size_t)q * bn + j0 + k) * 128 + vl);
                            r[k] = __float_as_uint(acc_v);
                        }
                        emit(r, j0, row0 + j0);
                    }
                    if (quarter == 0 && lane == 0) a.tail_ticket[grp] = 0;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, a.tmem_cols);
    }
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

bool lm_head_shape(int Mh, int smem_limit, LmShape* s) {
    if (Mh < 1 || Mh > 512) return false;
    if (Mh <= 256) {
        s->NB = 1;
        s->BN = (Mh + 15) / 16 * 16;
    } else {
        s->NB = 2;
        s->BN = ((Mh + 1) / 2 + 15) / 16 * 16;
    }
    const int cols = s->NB * s->BN;
    s->n_acc = (2 * cols <= 512) ? 2 : 1;
    const int need = s->n_acc * cols;
    uint32_t alloc = 32;
    while ((int)alloc < need) alloc <<= 1;
    s->tmem_cols = alloc;
    const int h_bytes = cols * 128;
    const int budget = smem_limit - 1024 - 512 - kEpiSmemBytes;  // slack, barriers, epilogue
    // hidden tiles are L2 hits: 3 stages; the rest of the budget deepens the
    // W ring (HBM latency under load is several microseconds)
    s->h_stages = 3;
    s->w_stages = (budget - s->h_stages * h_bytes) / kWStageBytes;
    if (s->w_stages > 16) s->w_stages = 16;
    if (s->w_stages < 4) {
        s->h_stages = 2;
        s->w_stages = (budget - s->h_stages * h_bytes) / kWStageBytes;
        if (s->w_stages > 16) s->w_stages = 16;
    }
    if (s->w_stages <= s->h_stages) return false;
    s->smem = (size_t)s->w_stages * kWStageBytes + (size_t)s->h_stages * h_bytes + kEpiSmemBytes +
              1024 + 512;
    return true;
}

void set_error_detail(const char* msg);

// pdl: launched as part of the whole step (programmatic dependent launch);
// counters_cleared: an earlier kernel of the step already cleared the
// left-over-tile counters in tail_ws.
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
    LmArgs a;
    a.w_rows = V < 128 ? V : 128;
    a.h_rows0 = Mh < sh.BN ? Mh : sh.BN;
    a.h_rows1 = sh.NB > 1 ? Mh - sh.BN : 0;
    CUtensorMap tw, th0, th1;
    if (!encode_bf16_2d(&tw, W, (uint64_t)V, (uint64_t)H, (uint32_t)a.w_rows)) {
        set_error_detail("lm_head: tensor map of W rejected");
        return cudaErrorInvalidValue;
    }
    if (!encode_bf16_2d(&th0, hidden, (uint64_t)Mh, (uint64_t)H, (uint32_t)a.h_rows0)) {
        set_error_detail("lm_head: tensor map of hidden rejected");
        return cudaErrorInvalidValue;
    }
    th1 = th0;
    if (sh.NB > 1 &&
        !encode_bf16_2d(&th1, hidden, (uint64_t)Mh, (uint64_t)H, (uint32_t)a.h_rows1)) {
        set_error_detail("lm_head: tensor map of hidden (second block) rejected");
        return cudaErrorInvalidValue;
    }
    a.V = V;
    a.Mh = Mh;
    a.H = H;
    a.BN = sh.BN;
    a.n_acc = sh.n_acc;
    a.w_stages = sh.w_stages;
    a.h_stages = sh.h_stages;
    a.n_tiles = (V + 127) / 128;
    a.tmem_cols = sh.tmem_cols;
    a.logits = logits;
    a.stats_part = stats_part;
    a.err_flag = err_flag;
    int grid = persistent_grid();
    if (grid > a.n_tiles) grid = a.n_tiles;
    // whole waves of tiles, then the left-over tiles split into row chunks
    a.n_full = (a.n_tiles / grid) * grid;
    const int left = a.n_tiles - a.n_full;
    a.tail_split = 1;
    a.tail_bn = 16;
    if (left > 0 && Mh >= 32) {
        int S = grid / left;
        const int max_chunks = (Mh + 15) / 16;
        if (S > max_chunks) S = max_chunks;
        if (S >= 2) {
            const int bn = ((Mh + S - 1) / S + 15) / 16 * 16;
            S = (Mh + bn - 1) / bn;
            if (S >= 2) {
                a.tail_split = S;
                a.tail_bn = bn;
            }
        }
    }
    // row chunks of at most 64 rows may also be split along K when CTAs are
    // still idle; the slices' partials and counters live in tail_ws
    a.tail_ksplit = 1;
    a.tail_part = nullptr;
    a.tail_ticket = nullptr;
    if (a.tail_split > 1 && a.tail_bn <= 64 && grid <= kMaxSMs && tail_ws) {
        int ks = grid / (left * a.tail_split);
        if (ks > 8) ks = 8;
        if (ks > H / 64) ks = H / 64;
        if (ks >= 2) {
            a.tail_ksplit = ks;
            a.tail_part = static_cast<float*>(tail_ws);
            a.tail_ticket = reinterpret_cast<int*>(static_cast<char*>(tail_ws) + kLmTailPartBytes);
            const cudaError_t me =
                counters_cleared ? cudaSuccess
                                 : cudaMemsetAsync(a.tail_ticket, 0, (size_t)left * a.tail_split * 4, st);
            if (me != cudaSuccess) {
                set_error_detail("lm_head: clearing the left-over tile counters");
                return me;
            }
        }
    }
    CUtensorMap tht = th0;
    if (a.tail_split > 1 &&
        !encode_bf16_2d(&tht, hidden, (uint64_t)Mh, (uint64_t)H, (uint32_t)a.tail_bn)) {
        set_error_detail("lm_head: tensor map of hidden (row chunks) rejected");
        return cudaErrorInvalidValue;
    }
    cudaError_t e = sh.NB == 1
        ? launch_kernel(pdl, lm_head_kernel<1>, dim3(grid), dim3(kLmThreads), sh.smem, st, tw, th0, th1, tht, a)
        : launch_kernel(pdl, lm_head_kernel<2>, dim3(grid), dim3(kLmThreads), sh.smem, st, tw, th0, th1, tht, a);
    if (e != cudaSuccess) set_error_detail("lm_head: launch failed");
    return e;
}

}  // namespace isd
