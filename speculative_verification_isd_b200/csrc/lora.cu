// R-ISD gated LoRA on the MASK rows (a3): h' = bf16(h + bf16(h A) B).
//
// Residual ISD adds a rank-r gated adapter that is active at MASK positions
// only, while verify positions keep the base weights ("自省扩散语言模型的 token
// 生成机制与工程实践", section "Token 生成的核心参数与验收机制"; the I-DLM project
// page's R-ISD paragraph).  Here it is applied to the hidden state that feeds
// the LM head.  The work is two thin GEMMs (at B=64, N=4: 192 rows x 4096 x
// 128 and back), about 0.4 GFLOP, done on mma.sync tiles:
//   1. T_part[z] = H_mask . A over K-slice z (fp32, split-K for parallelism)
//   2. T = bf16(sum_z T_part[z]) in slice order
//   3. h' = bf16(h + T . B) on the MASK rows, h' = h copied on the clean rows
//      (a second plane of the grid, so no separate copy of hidden).
// The kernels wait for their predecessor when launched as dependents (pdl).
#include "common.cuh"
#include "plan.h"
#include "launch.h"

namespace isd {

constexpr int kLBM = 64, kLBN = 64, kLBK = 32;
constexpr int kAStride = kLBK + 8;  // padded smem rows (bf16): conflict-free ldmatrix
constexpr int kBStride = kLBN + 8;

struct LoraGemmArgs {
    int rows;             // MASK rows = B * (N-1)
    int N, Q, H, r;
    int K, ncols;         // reduction length and output columns of this GEMM
    int k_per_split;      // multiple of kLBK
    const __nv_bfloat16* a_src;  // mode 0: hidden [M,H]; mode 1: T [rows, r]
    const __nv_bfloat16* bmat;   // [K, ncols] row-major
    float* part;                 // mode 0 output [ksplit][rows][r]
    const __nv_bfloat16* hidden; // mode 1 addend
    __nv_bfloat16* out;          // mode 1 output (hidden' [M,H])
    int clean_rows;              // mode 1: B * N rows copied by the grid's second plane
};

// Row of the A operand for logical row m.
template <int MODE>
ISD_DEVINL const __nv_bfloat16* lora_a_row(const LoraGemmArgs& g, int m) {
    if (MODE == 0) {
        const int b = m / (g.N - 1), mm = m % (g.N - 1);
        return g.a_src + ((size_t)b * g.Q + g.N + mm) * g.H;
    }
    return g.a_src + (size_t)m * g.r;
}

template <int MODE>
__global__ void __launch_bounds__(128) lora_gemm_kernel(const __grid_constant__ LoraGemmArgs g) {
    __shared__ __align__(16) __nv_bfloat16 As[2][kLBM * kAStride];
    __shared__ __align__(16) __nv_bfloat16 Bs[2][kLBK * kBStride];
    pdl_trigger();
    pdl_wait();  // hidden (attention) or T (the first kernel) comes from the preceding kernel
    const int m0 = blockIdx.x * kLBM, n0 = blockIdx.y * kLBN, z = blockIdx.z;
    if (MODE == 1 && z == 1) {
        // clean rows: h' = h, 64 columns of 64 rows, 16 bytes per thread and step
        for (int i = threadIdx.x; i < kLBM * (kLBN / 8); i += 128) {
            const int cr = m0 + i / (kLBN / 8), c8 = (i % (kLBN / 8)) * 8;
            if (cr >= g.clean_rows || n0 + c8 >= g.H) continue;
            const int b = cr / g.N, s = cr % g.N;
            const size_t off = ((size_t)b * g.Q + s) * g.H + n0 + c8;
            *reinterpret_cast<uint4*>(g.out + off) = *reinterpret_cast<const uint4*>(g.hidden + off);
        }
        return;
    }
    if (m0 >= g.rows) return;
    const int kbeg = z * g.k_per_split;
    const int kend = min(g.K, kbeg + g.k_per_split);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int wm = warp >> 1, wn = warp & 1;

    auto load = [&](int buf, int k0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int ci = tid + i * 128;
            const int r = ci >> 2, c = ci & 3;
            const int m = m0 + r;
            const void* src = g.bmat;
            int bytes = 0;
            if (m < g.rows) {
                src = lora_a_row<MODE>(g, m) + k0 + c * 8;
                bytes = 16;
            }
            cp_async16(smem_u32(&As[buf][r * kAStride + c * 8]), src, bytes);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int ci = tid + i * 128;
            const int k = ci >> 3, c = ci & 7;
            const int n = n0 + c * 8;
            const void* src = g.bmat;
            int bytes = 0;
            if (n < g.ncols) {
                src = g.bmat + (size_t)(k0 + k) * g.ncols + n;
                bytes = 16;
            }
            cp_async16(smem_u32(&Bs[buf][k * kBStride + c * 8]), src, bytes);
        }
    };

    float acc[2][4][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

    const int nk = (kend - kbeg) / kLBK;
    if (nk > 0) load(0, kbeg);
    cp_async_commit();
    for (int it = 0; it < nk; ++it) {
        if (it + 1 < nk) load((it + 1) & 1, kbeg + (it + 1) * kLBK);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const int buf = it & 1;
#pragma unroll
        for (int kk = 0; kk < kLBK; kk += 16) {
            uint32_t af[2][4];
            const int j = lane >> 3;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int r = wm * 32 + mt * 16 + (j & 1) * 8 + (lane & 7);
                ldmatrix_x4(af[mt], smem_u32(&As[buf][r * kAStride + kk + (j >> 1) * 8]));
            }
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bf[4];
                const int k = kk + (j & 1) * 8 + (lane & 7);
                ldmatrix_x4_trans(bf, smem_u32(&Bs[buf][k * kBStride + wn * 32 + np * 16 + (j >> 1) * 8]));
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    mma_bf16_16816(acc[mt][np * 2], af[mt], bf[0], bf[1]);
                    mma_bf16_16816(acc[mt][np * 2 + 1], af[mt], bf[2], bf[3]);
                }
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();

#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int m = m0 + wm * 32 + mt * 16 + (lane >> 2) + h * 8;
                const int n = n0 + wn * 32 + nt * 8 + (lane & 3) * 2;
                if (m >= g.rows || n >= g.ncols) continue;
                const float v0 = acc[mt][nt][h * 2], v1 = acc[mt][nt][h * 2 + 1];
                if (MODE == 0) {
                    *reinterpret_cast<float2*>(g.part + ((size_t)z * g.rows + m) * g.r + n) =
                        make_float2(v0, v1);
                } else {
                    const int b = m / (g.N - 1), mm = m % (g.N - 1);
                    const size_t off = ((size_t)b * g.Q + g.N + mm) * g.H + n;
                    const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162*>(g.hidden + off);
                    const float2 hf = __bfloat1622float2(h2);
                    *reinterpret_cast<__nv_bfloat162*>(g.out + off) =
                        __floats2bfloat162_rn(hf.x + v0, hf.y + v1);
                }
            }
}

// T[m][n] = bf16(sum_z part[z][m][n]) in z order.
__global__ void lora_reduce_kernel(const float* __restrict__ part, int ksplit, int count,
                                   __nv_bfloat16* __restrict__ t) {
    pdl_trigger();
    pdl_wait();  // the partials come from the preceding kernel
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= count) return;
    float s = 0.f;
    for (int z = 0; z < ksplit; ++z) s += part[(size_t)z * count + i];
    t[i] = __float2bfloat16_rn(s);
}

// hidden' = hidden with the adapter applied to the MASK rows (pdl: launch the
// kernels as programmatic dependents of the preceding ones).
cudaError_t launch_lora(const Plan& p, const isd_dims* d, const uint16_t* hidden,
                        const uint16_t* lora_A, const uint16_t* lora_B, uint16_t* hidden_out,
                        void* ws, cudaStream_t st, bool pdl) {
    char* w = static_cast<char*>(ws);
    cudaError_t e = cudaSuccess;
    const int r = d->lora_rank;
    LoraGemmArgs g = {};
    g.rows = p.lora_rows;
    g.N = d->N;
    g.Q = p.Q;
    g.H = p.H;
    g.r = r;
    g.clean_rows = d->B * d->N;
    float* part = reinterpret_cast<float*>(w + p.off_lora_part);
    __nv_bfloat16* t = reinterpret_cast<__nv_bfloat16*>(w + p.off_lora_t);
    if (p.lora_rows > 0) {
        // 1. partial h.A
        const int kiters = p.H / kLBK;
        const int per = (kiters + p.lora_ksplit - 1) / p.lora_ksplit;
        g.K = p.H;
        g.ncols = r;
        g.k_per_split = per * kLBK;
        g.a_src = reinterpret_cast<const __nv_bfloat16*>(hidden);
        g.bmat = reinterpret_cast<const __nv_bfloat16*>(lora_A);
        g.part = part;
        const int ks = (kiters + per - 1) / per;
        dim3 g1((g.rows + kLBM - 1) / kLBM, (r + kLBN - 1) / kLBN, ks);
        if ((e = launch_kernel(pdl, lora_gemm_kernel<0>, g1, dim3(128), 0, st, g)) != cudaSuccess)
            return e;
        // 2. fixed-order reduction, rounded to bf16
        const int count = g.rows * r;
        if ((e = launch_kernel(pdl, lora_reduce_kernel, dim3((count + 255) / 256), dim3(256), 0, st,
                               (const float*)part, ks, count, t)) != cudaSuccess)
            return e;
    }
    // 3. h' = bf16(h + T.B) on the MASK rows (plane 0), h' = h on the clean rows (plane 1)
    g.K = r;
    g.ncols = p.H;
    g.k_per_split = r;
    g.a_src = t;
    g.bmat = reinterpret_cast<const __nv_bfloat16*>(lora_B);
    g.part = nullptr;
    g.hidden = reinterpret_cast<const __nv_bfloat16*>(hidden);
    g.out = reinterpret_cast<__nv_bfloat16*>(hidden_out);
    const int mtiles = (max(g.rows, g.clean_rows) + kLBM - 1) / kLBM;
    dim3 g2(mtiles, (p.H + kLBN - 1) / kLBN, 2);
    return launch_kernel(pdl, lora_gemm_kernel<1>, g2, dim3(128), 0, st, g);
}

}  // namespace isd
