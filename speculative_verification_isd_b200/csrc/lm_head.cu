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
//  * every mbarrier wait is bounded (about 2 s); on time-out the CTA raises
//    ISD_FLAG_WAIT_TIMEOUT, every role leaves its loop, outstanding TMA loads
//    and MMAs are drained with bounded waits, and TMEM is released.
#include <cuda.h>

#include "common.cuh"
#include "plan.h"
#include "sm100.cuh"

namespace isd {

struct LmArgs {
    int V, Mh, H;
    int BN, NB, n_acc, stages, n_tiles;
    int w_rows, h_rows0, h_rows1;  // TMA box heights (never taller than the tensor)
    uint32_t tmem_cols;
    float* logits;
    int32_t* err_flag;
};

constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kLmThreads = 192;

__global__ void __launch_bounds__(kLmThreads, 1)
lm_head_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_h0,
               const __grid_constant__ CUtensorMap tmap_h1, LmArgs a) {
    using namespace sm100;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int b_bytes = a.NB * a.BN * 128;
    const int stage_bytes = 16384 + b_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)a.stages * stage_bytes);
    uint64_t* empty = full + a.stages;
    uint64_t* tfull = empty + a.stages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    __shared__ int never;  // a flag nothing sets: used by the final drains

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(&full[s], 1);
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
        if (a.NB > 1) prefetch_tmap(&tmap_h1);
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
    // Every CTA streams its own rows of W but all of them read the same
    // hidden tile; starting each CTA's K loop at a different block spreads
    // those reads over the L2 slices instead of hitting one slice from 148 SMs.
    const int kb0 = (int)(blockIdx.x % (unsigned)kblocks);

    auto give_up = [&]() {
        *abort_flag = 1;
        raise_flag(a.err_flag, ISD_FLAG_WAIT_TIMEOUT);
    };

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_h = policy_evict_last();
            uint32_t armed = 0, parity_bits = 0;
            int it = 0;
            // rows of a box beyond the tensor are not delivered (and not used:
            // their accumulator columns / vocabulary rows are never stored)
            const uint32_t tx = (uint32_t)(a.w_rows + a.h_rows0 + a.h_rows1) * 128u;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x) {
                for (int j = 0; j < kblocks; ++j, ++it) {
                    const int kb = (j + kb0) % kblocks;
                    const int s = it % a.stages;
                    const uint32_t round = (uint32_t)(it / a.stages);
                    if (!mbar_wait_bounded(&empty[s], (round & 1) ^ 1, abort_flag, kWaitLimitNs)) {
                        give_up();
                        ok = false;
                        break;
                    }
                    unsigned char* sa = smem + (size_t)s * stage_bytes;
                    unsigned char* sb = sa + 16384;
                    mbar_arrive_expect_tx(&full[s], tx);
                    tma_load_2d(sa, &tmap_w, &full[s], kb * 64, tile * 128, pol_w);
                    tma_load_2d(sb, &tmap_h0, &full[s], kb * 64, 0, pol_h);
                    if (a.NB > 1)
                        tma_load_2d(sb + a.BN * 128, &tmap_h1, &full[s], kb * 64, a.BN, pol_h);
                    armed |= 1u << s;
                    parity_bits = (parity_bits & ~(1u << s)) | ((round & 1) << s);
                }
            }
            // no TMA write may land after this CTA leaves: wait for every
            // stage's last armed phase
            for (int s = 0; s < a.stages; ++s)
                if (armed >> s & 1)
                    mbar_wait_bounded(&full[s], parity_bits >> s & 1, &never, kWaitLimitNs);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            const uint32_t idesc = idesc_bf16_f32(128, a.BN);
            int it = 0, lt = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x, ++lt) {
                const int acc = lt % a.n_acc;
                const uint32_t use = (uint32_t)(lt / a.n_acc);
                if (!mbar_wait_bounded(&tempty[acc], (use & 1) ^ 1, abort_flag, kWaitLimitNs)) {
                    give_up();
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(acc * a.NB * a.BN);
                for (int j = 0; j < kblocks; ++j, ++it) {
                    const int s = it % a.stages;
                    const uint32_t round = (uint32_t)(it / a.stages);
                    if (!mbar_wait_bounded(&full[s], round & 1, abort_flag, kWaitLimitNs)) {
                        give_up();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + (size_t)s * stage_bytes);
                    const uint32_t sb = sa + 16384;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t adesc = smem_desc_sw128(sa + k * 32);
                        for (int nb = 0; nb < a.NB; ++nb) {
                            const uint64_t bdesc = smem_desc_sw128(sb + nb * a.BN * 128 + k * 32);
                            mma_f16_ss(d0 + nb * a.BN, adesc, bdesc, idesc, (j | k) != 0);
                        }
                    }
                    mma_commit(&empty[s]);
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
        int lt = 0;
        for (int tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x, ++lt) {
            const int acc = lt % a.n_acc;
            const uint32_t use = (uint32_t)(lt / a.n_acc);
            int ok = 1;
            if (lane == 0) {
                ok = mbar_wait_bounded(&tfull[acc], use & 1, abort_flag, kWaitLimitNs);
                if (!ok) give_up();
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const int v = tile * 128 + quarter * 32 + lane;
            const bool v_ok = v < a.V;
            const uint32_t taddr =
                tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * a.NB * a.BN);
            for (int nb = 0; nb < a.NB; ++nb) {
                for (int j0 = 0; j0 < a.BN; j0 += 32) {
                    uint32_t r[32];
                    // BN is a multiple of 16: the tail is one 16-column load,
                    // so no load reaches past the allocated columns
                    if (a.BN - j0 >= 32)
                        tmem_ld_32x32b_x32(taddr + nb * a.BN + j0, r);
                    else
                        tmem_ld_32x32b_x16(taddr + nb * a.BN + j0, r);
                    tmem_ld_wait();
                    const int mbase = nb * a.BN + j0;
                    if (v_ok) {
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const int m = mbase + k;
                            if (j0 + k < a.BN && m < a.Mh)
                                a.logits[(size_t)m * a.V + v] = __uint_as_float(r[k]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
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
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

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
    int BN, NB, n_acc, stages;
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
    const int stage_bytes = 16384 + cols * 128;
    const int budget = smem_limit - 1024 - 256;  // alignment slack + barriers
    s->stages = budget / stage_bytes;
    if (s->stages > 8) s->stages = 8;
    if (s->stages < 2) return false;
    s->smem = (size_t)s->stages * stage_bytes + 1024 + 256;
    return true;
}

static int num_sms_of_current_device() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

void set_error_detail(const char* msg);

cudaError_t launch_lm_head(const uint16_t* hidden, const uint16_t* W, int Mh, int H, int V,
                           float* logits, int32_t* err_flag, cudaStream_t st) {
    // dynamic shared memory available to this kernel on the current device
    static int smem_limit_dev[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!smem_limit_dev[dev]) {
        int optin = 0;
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, lm_head_kernel) != cudaSuccess) {
            set_error_detail("lm_head: kernel attributes unavailable");
            return cudaErrorInvalidValue;
        }
        const int limit = optin - (int)fa.sharedSizeBytes;
        if (cudaFuncSetAttribute(lm_head_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
    a.NB = sh.NB;
    a.n_acc = sh.n_acc;
    a.stages = sh.stages;
    a.n_tiles = (V + 127) / 128;
    a.tmem_cols = sh.tmem_cols;
    a.logits = logits;
    a.err_flag = err_flag;
    int grid = num_sms_of_current_device();
    if (grid > a.n_tiles) grid = a.n_tiles;
    lm_head_kernel<<<grid, kLmThreads, sh.smem, st>>>(tw, th0, th1, a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) set_error_detail("lm_head: launch failed");
    return e;
}

}  // namespace isd
