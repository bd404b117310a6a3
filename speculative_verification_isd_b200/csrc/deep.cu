// Full-depth synthetic I-DLM forward over the ISD block: the decoder stack
// that the single-layer step stands in for.
//
// I-DLM keeps the autoregressive model's stack and serving path
// ("I-DLM：扩散模型如何用“自省一致性”追上自回归模型质量", section
// "推理：复用 AR 推理栈"), and the pages' 8B model is built from Qwen3-8B.  The
// layer internals are not in the pages; this is the base model's decoder
// layer, run over all 2N-1 slots of the block in one pass:
//   x += O(attn(RoPE(qk_norm(QKV(rmsnorm(x))))))
//   x += down(silu(gate(h)) * up(h)),  h = rmsnorm(x)
// with the ISD slot layout and strict-causal mask of the single-layer step
// at every layer (each layer has its own paged K/V pool under one page
// table), and the final RMSNorm before the LM head.
//
// Rounding points: every RMSNorm output, every GEMM output (the O and down
// projections add the residual before that rounding), q and k after their
// norm and rotation, the attention output, silu(gate) * up.  Between two
// rounding points the arithmetic is fp32.
//
// The four projections are plain dense GEMMs (M = B*(2N-1) rows against
// weights that stream once per step); they run on cuBLASLt (bf16 in/out,
// fp32 accumulation, the residual as C with beta = 1).  The norms, the
// q/k rotation, the activation and the attention are this library's kernels.
#include <cublasLt.h>
#include <cuda_bf16.h>
#include <stdio.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "plan.h"

namespace isd {

void set_error_detail(const char* msg);

constexpr int kNormThreads = 256;

// y = bf16(x / sqrt(mean(x^2) + eps) * w) per row of H (H % 8 == 0).
__global__ void __launch_bounds__(kNormThreads)
rmsnorm_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w,
               __nv_bfloat16* __restrict__ y, int H, float eps) {
    const int row = blockIdx.x;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)row * H);
    const int n8 = H / 8;
    float ss = 0.f;
    for (int i = threadIdx.x; i < n8; i += kNormThreads) {
        const uint4 v = xr[i];
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(p[e]);
            ss = fmaf(f.x, f.x, ss);
            ss = fmaf(f.y, f.y, ss);
        }
    }
    __shared__ float red[kNormThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int k = 0; k < kNormThreads / 32; ++k) tot += red[k];
    const float r = __frsqrt_rn(tot / (float)H + eps);
    const uint4* wr = reinterpret_cast<const uint4*>(w);
    uint4* yr = reinterpret_cast<uint4*>(y + (size_t)row * H);
    for (int i = threadIdx.x; i < n8; i += kNormThreads) {
        const uint4 v = xr[i], wv = __ldg(wr + i);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
        const __nv_bfloat162* q = reinterpret_cast<const __nv_bfloat162*>(&wv);
        uint4 o;
        __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(p[e]), g = __bfloat1622float2(q[e]);
            po[e] = __floats2bfloat162_rn(f.x * r * g.x, f.y * r * g.y);
        }
        yr[i] = o;
    }
}

// Per head of one block row: q and k heads are RMS-normalised over D (weights
// q_norm / k_norm), rotated by the slot's position (rotate-half pairs, table
// rows (cos, sin)) and rounded once; v heads are copied.  A head takes
// L = D/8 lanes (two heads per warp at D = 128, four at D = 64); lane j of a
// head holds elements 4j..4j+3 and their rotation partners 4j+D/2..4j+D/2+3
// (8-byte loads), so the rotation needs no exchange between lanes.
template <int D>
__global__ void __launch_bounds__(256)
qk_norm_rope_kernel(const __nv_bfloat16* __restrict__ qkv, const __nv_bfloat16* __restrict__ q_norm,
                    const __nv_bfloat16* __restrict__ k_norm, const float2* __restrict__ rope,
                    int rope_len, const int32_t* __restrict__ kv_len,
                    const int32_t* __restrict__ n_clean, int N, int Q, int Hq, int Hkv, float eps,
                    __nv_bfloat16* __restrict__ q_out, __nv_bfloat16* __restrict__ k_out,
                    __nv_bfloat16* __restrict__ v_out, int32_t* err_flag) {
    constexpr int L = D / 8;           // lanes per head (4 elements of each half each)
    constexpr int HPW = 32 / L;        // heads per warp and pass
    const int row = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / L, j = lane % L;
    const int b = row / Q, s = row - b * Q;
    const int kv = max(kv_len[b], 0), c = n_clean[b];
    int pos = s < N ? kv + s : kv + c + (s - N);
    pos = max(pos, 0);  // a bad n_clean is flagged by the attention that follows
    if (pos >= rope_len) {
        if (threadIdx.x == 0) raise_flag(err_flag, ISD_FLAG_CAPACITY);
        pos = rope_len - 1;
    }
    const float2* cs = rope + (size_t)pos * (D / 2) + 4 * j;
    const int heads = Hq + 2 * Hkv;
    const __nv_bfloat16* src = qkv + (size_t)row * heads * D;
    for (int h0 = warp * HPW; h0 < heads; h0 += 8 * HPW) {
        const int h = h0 + sub;
        const bool live = h < heads;
        uint2 lo = make_uint2(0, 0), hi = make_uint2(0, 0);
        if (live) {
            lo = *reinterpret_cast<const uint2*>(src + h * D + 4 * j);
            hi = *reinterpret_cast<const uint2*>(src + h * D + D / 2 + 4 * j);
        }
        if (live && h >= Hq + Hkv) {
            __nv_bfloat16* dst = v_out + ((size_t)row * Hkv + (h - Hq - Hkv)) * D;
            *reinterpret_cast<uint2*>(dst + 4 * j) = lo;
            *reinterpret_cast<uint2*>(dst + D / 2 + 4 * j) = hi;
        }
        const bool is_q = h < Hq;
        const __nv_bfloat162* pl = reinterpret_cast<const __nv_bfloat162*>(&lo);
        const __nv_bfloat162* ph = reinterpret_cast<const __nv_bfloat162*>(&hi);
        float x[4], y[4];
        {
            const float2 a0 = __bfloat1622float2(pl[0]), a1 = __bfloat1622float2(pl[1]);
            const float2 b0 = __bfloat1622float2(ph[0]), b1 = __bfloat1622float2(ph[1]);
            x[0] = a0.x; x[1] = a0.y; x[2] = a1.x; x[3] = a1.y;
            y[0] = b0.x; y[1] = b0.y; y[2] = b1.x; y[3] = b1.y;
        }
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) ss = fmaf(y[e], y[e], fmaf(x[e], x[e], ss));
        // sum over the head's L lanes (an aligned group of the warp)
#pragma unroll
        for (int o = L / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (!live || h >= Hq + Hkv) continue;
        const float r = __frsqrt_rn(ss / (float)D + eps);
        const __nv_bfloat16* wn = is_q ? q_norm : k_norm;
        const uint2 wl = __ldg(reinterpret_cast<const uint2*>(wn + 4 * j));
        const uint2 wh = __ldg(reinterpret_cast<const uint2*>(wn + D / 2 + 4 * j));
        const __nv_bfloat162* pwl = reinterpret_cast<const __nv_bfloat162*>(&wl);
        const __nv_bfloat162* pwh = reinterpret_cast<const __nv_bfloat162*>(&wh);
        const float2 w0 = __bfloat1622float2(pwl[0]), w1 = __bfloat1622float2(pwl[1]);
        const float2 v0 = __bfloat1622float2(pwh[0]), v1 = __bfloat1622float2(pwh[1]);
        const float wlo[4] = {w0.x, w0.y, w1.x, w1.y}, whi[4] = {v0.x, v0.y, v1.x, v1.y};
        float olo[4], ohi[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 t = __ldg(cs + e);
            const float l = x[e] * r * wlo[e], u = y[e] * r * whi[e];
            olo[e] = l * t.x - u * t.y;
            ohi[e] = u * t.x + l * t.y;
        }
        __nv_bfloat16* dst = is_q ? q_out + ((size_t)row * Hq + h) * D
                                  : k_out + ((size_t)row * Hkv + (h - Hq)) * D;
        uint2 ol, oh;
        reinterpret_cast<__nv_bfloat162*>(&ol)[0] = __floats2bfloat162_rn(olo[0], olo[1]);
        reinterpret_cast<__nv_bfloat162*>(&ol)[1] = __floats2bfloat162_rn(olo[2], olo[3]);
        reinterpret_cast<__nv_bfloat162*>(&oh)[0] = __floats2bfloat162_rn(ohi[0], ohi[1]);
        reinterpret_cast<__nv_bfloat162*>(&oh)[1] = __floats2bfloat162_rn(ohi[2], ohi[3]);
        *reinterpret_cast<uint2*>(dst + 4 * j) = ol;
        *reinterpret_cast<uint2*>(dst + D / 2 + 4 * j) = oh;
    }
}

// act = bf16(silu(gate) * up) from gate_up [M, 2I] (gate columns first).
__global__ void __launch_bounds__(256)
silu_mul_kernel(const __nv_bfloat16* __restrict__ gu, __nv_bfloat16* __restrict__ act, int M,
                int I) {
    const int n8 = I / 8;
    const size_t total = (size_t)M * n8;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t row = i / n8, j = i - row * n8;
        const uint4 g = reinterpret_cast<const uint4*>(gu + row * 2 * I)[j];
        const uint4 u = reinterpret_cast<const uint4*>(gu + row * 2 * I + I)[j];
        const __nv_bfloat162* pg = reinterpret_cast<const __nv_bfloat162*>(&g);
        const __nv_bfloat162* pu = reinterpret_cast<const __nv_bfloat162*>(&u);
        uint4 o;
        __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 a = __bfloat1622float2(pg[e]), v = __bfloat1622float2(pu[e]);
            const float sa = a.x / (1.f + expf(-a.x)), sb = a.y / (1.f + expf(-a.y));
            po[e] = __floats2bfloat162_rn(sa * v.x, sb * v.y);
        }
        reinterpret_cast<uint4*>(act + row * I)[j] = o;
    }
}

// Block embeddings: slot s of request b takes row id of E [V+1, H] (its
// clean token for an active clean slot, the MASK row V otherwise), 16 bytes
// per thread.
__global__ void __launch_bounds__(256)
embed_block_kernel(const __nv_bfloat16* __restrict__ E, const int32_t* __restrict__ n_clean,
                   const int32_t* __restrict__ clean_tok, int N, int Q, int V, int H,
                   __nv_bfloat16* __restrict__ x, int32_t* err_flag) {
    const int s = blockIdx.x, b = blockIdx.y;
    const int c = n_clean[b];
    int id = V;
    if (s < N && s < c && c <= N) {
        const int t = clean_tok[(size_t)b * N + s];
        if (t >= 0 && t < V) id = t;
        else if (threadIdx.x == 0) raise_flag(err_flag, ISD_FLAG_TOKEN_OOB);
    }
    const uint4* src = reinterpret_cast<const uint4*>(E + (size_t)id * H);
    uint4* dst = reinterpret_cast<uint4*>(x + ((size_t)b * Q + s) * H);
    for (int i = threadIdx.x; i < H / 8; i += 256) dst[i] = __ldg(src + i);
}

cudaError_t launch_embed_block(const isd_dims* d, int Q, const void* E, const int32_t* n_clean,
                               const int32_t* clean_tok, void* x, int32_t* err_flag,
                               cudaStream_t st) {
    embed_block_kernel<<<dim3(Q, d->B), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(E), n_clean, clean_tok, d->N, Q, d->V,
        d->Hq * d->D, reinterpret_cast<__nv_bfloat16*>(x), err_flag);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// cuBLASLt: Y[M, Nout] (+)= X[M, K] . W[Nout, K]^T, bf16 in/out, fp32 compute.
// Column-major view: Y^T (Nout x M) = W (op T) x X^T.  Descriptors and the
// algorithm are cached per shape, the handle per device.  The algorithm: on
// the first call for a shape (outside stream capture), the heuristic's best
// few candidates are each timed on the call's own operands, writing into a
// scratch output, and the fastest is kept; under capture, the heuristic's
// first choice.
// ---------------------------------------------------------------------------
namespace {
struct GemmPlan {
    int dev, M, Nout, K, acc;
    size_t ws;
    cublasLtMatmulDesc_t op;
    cublasLtMatrixLayout_t a, b, c;
    cublasLtMatmulAlgo_t algo;
};
constexpr int kMaxGemmPlans = 64;
GemmPlan g_plans[kMaxGemmPlans];
int g_nplans = 0;
cublasLtHandle_t g_lt[64];
std::mutex g_plan_mutex;  // the handle and plan caches are shared by all host threads

cublasLtHandle_t lt_handle(int dev) {
    if (dev < 0 || dev >= 64) return nullptr;
    if (!g_lt[dev] && cublasLtCreate(&g_lt[dev]) != CUBLAS_STATUS_SUCCESS) g_lt[dev] = nullptr;
    return g_lt[dev];
}

constexpr int kTuneCandidates = 8;

// Mean time of `reps` runs of one candidate (ms), or a negative value if it fails.
float time_algo(cublasLtHandle_t h, const GemmPlan& p, const cublasLtMatmulAlgo_t& algo,
                const void* X, const void* W, void* scratch, void* lt_ws, size_t ws,
                cudaStream_t st) {
    const float alpha = 1.f, beta = 0.f;
    auto run = [&]() {
        return cublasLtMatmul(h, p.op, &alpha, W, p.a, X, p.b, &beta, scratch, p.c, scratch, p.c,
                              &algo, lt_ws, ws, st);
    };
    if (run() != CUBLAS_STATUS_SUCCESS) return -1.f;
    cudaEvent_t e0, e1;
    if (cudaEventCreate(&e0) != cudaSuccess) return -1.f;
    if (cudaEventCreate(&e1) != cudaSuccess) {
        cudaEventDestroy(e0);
        return -1.f;
    }
    constexpr int reps = 3;
    float ms = -1.f;
    bool ok = cudaEventRecord(e0, st) == cudaSuccess;
    for (int r = 0; ok && r < reps; ++r) ok = run() == CUBLAS_STATUS_SUCCESS;
    if (ok && cudaEventRecord(e1, st) == cudaSuccess && cudaEventSynchronize(e1) == cudaSuccess &&
        cudaEventElapsedTime(&ms, e0, e1) == cudaSuccess)
        ms /= reps;
    else
        ms = -1.f;
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    return ms;
}

const GemmPlan* gemm_plan(int dev, int M, int Nout, int K, bool acc, size_t ws, const void* X,
                          const void* W, void* scratch, size_t scratch_bytes, void* lt_ws,
                          cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(g_plan_mutex);
    for (int i = 0; i < g_nplans; ++i) {
        const GemmPlan& p = g_plans[i];
        if (p.dev == dev && p.M == M && p.Nout == Nout && p.K == K && p.acc == (int)acc && p.ws == ws)
            return &p;
    }
    if (g_nplans == kMaxGemmPlans) return nullptr;  // more shapes than the cache holds
    cublasLtHandle_t h = lt_handle(dev);
    if (!h) return nullptr;
    GemmPlan p{dev, M, Nout, K, (int)acc, ws};
    const cublasOperation_t ta = CUBLAS_OP_T, tb = CUBLAS_OP_N;
    if (cublasLtMatmulDescCreate(&p.op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS)
        return nullptr;
    cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof(ta));
    cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof(tb));
    cublasLtMatrixLayoutCreate(&p.a, CUDA_R_16BF, K, Nout, K);
    cublasLtMatrixLayoutCreate(&p.b, CUDA_R_16BF, K, M, K);
    cublasLtMatrixLayoutCreate(&p.c, CUDA_R_16BF, Nout, M, Nout);
    cublasLtMatmulPreference_t pref;
    cublasLtMatmulPreferenceCreate(&pref);
    cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws,
                                         sizeof(ws));
    cublasLtMatmulHeuristicResult_t res[kTuneCandidates];
    int n = 0;
    const cublasStatus_t st = cublasLtMatmulAlgoGetHeuristic(h, p.op, p.a, p.b, p.c, p.c, pref,
                                                             kTuneCandidates, res, &n);
    cublasLtMatmulPreferenceDestroy(pref);
    if (st != CUBLAS_STATUS_SUCCESS || n < 1) return nullptr;
    p.algo = res[0].algo;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    const bool capturing = cudaStreamIsCapturing(stream, &cap) != cudaSuccess ||
                           cap != cudaStreamCaptureStatusNone;
    if (n > 1 && !capturing && scratch && scratch_bytes >= (size_t)M * Nout * 2) {
        float best = -1.f;
        for (int i = 0; i < n; ++i) {
            if (res[i].state != CUBLAS_STATUS_SUCCESS || res[i].workspaceSize > ws) continue;
            const float t = time_algo(h, p, res[i].algo, X, W, scratch, lt_ws, ws, stream);
            if (t > 0.f && (best < 0.f || t < best)) {
                best = t;
                p.algo = res[i].algo;
            }
        }
        cudaGetLastError();  // a failed candidate leaves no sticky error
    }
    g_plans[g_nplans] = p;
    return &g_plans[g_nplans++];
}
}  // namespace

// scratch: scratch_bytes of device memory the first call for a shape may
// overwrite while it times the candidates (not an operand of this call).
cudaError_t gemm_bf16(int M, int Nout, int K, const void* X, const void* W, void* Y, bool acc,
                      void* lt_ws, size_t lt_ws_bytes, void* scratch, size_t scratch_bytes,
                      cudaStream_t st) {
    int dev = 0;
    cudaGetDevice(&dev);
    const GemmPlan* p = gemm_plan(dev, M, Nout, K, acc, lt_ws_bytes, X, W, scratch, scratch_bytes,
                                  lt_ws, st);
    if (!p) {
        set_error_detail("cuBLASLt: no bf16 GEMM plan for this shape (no algorithm, or 64 shapes cached)");
        return cudaErrorNotSupported;
    }
    cublasLtHandle_t h;
    {
        std::lock_guard<std::mutex> lock(g_plan_mutex);
        h = g_lt[dev];
    }
    const float alpha = 1.f, beta = acc ? 1.f : 0.f;
    const cublasStatus_t s = cublasLtMatmul(h, p->op, &alpha, W, p->a, X, p->b, &beta,
                                            Y, p->c, Y, p->c, &p->algo, lt_ws, lt_ws_bytes, st);
    if (s != CUBLAS_STATUS_SUCCESS) {
        char msg[96];
        snprintf(msg, sizeof(msg), "cuBLASLt matmul failed (status %d)", (int)s);
        set_error_detail(msg);
        return cudaErrorLaunchFailure;
    }
    return cudaGetLastError();
}

cudaError_t launch_rmsnorm(const void* x, const void* w, void* y, int M, int H, float eps,
                           cudaStream_t st) {
    rmsnorm_kernel<<<M, kNormThreads, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(x),
                                               reinterpret_cast<const __nv_bfloat16*>(w),
                                               reinterpret_cast<__nv_bfloat16*>(y), H, eps);
    return cudaGetLastError();
}

cudaError_t launch_qk_norm_rope(const isd_dims* d, int Q, const void* qkv, const void* q_norm,
                                const void* k_norm, const float* rope, int rope_len,
                                const int32_t* kv_len, const int32_t* n_clean, float eps, void* q,
                                void* k, void* v, int32_t* err_flag, cudaStream_t st) {
    const int M = d->B * Q;
    const auto* a = reinterpret_cast<const __nv_bfloat16*>(qkv);
    const auto* qn = reinterpret_cast<const __nv_bfloat16*>(q_norm);
    const auto* kn = reinterpret_cast<const __nv_bfloat16*>(k_norm);
    const auto* cs = reinterpret_cast<const float2*>(rope);
    auto* qo = reinterpret_cast<__nv_bfloat16*>(q);
    auto* ko = reinterpret_cast<__nv_bfloat16*>(k);
    auto* vo = reinterpret_cast<__nv_bfloat16*>(v);
    if (d->D == 128)
        qk_norm_rope_kernel<128><<<M, 256, 0, st>>>(a, qn, kn, cs, rope_len, kv_len, n_clean, d->N,
                                                    Q, d->Hq, d->Hkv, eps, qo, ko, vo, err_flag);
    else
        qk_norm_rope_kernel<64><<<M, 256, 0, st>>>(a, qn, kn, cs, rope_len, kv_len, n_clean, d->N,
                                                   Q, d->Hq, d->Hkv, eps, qo, ko, vo, err_flag);
    return cudaGetLastError();
}

cudaError_t launch_silu_mul(const void* gu, void* act, int M, int I, cudaStream_t st) {
    const size_t total = (size_t)M * (I / 8);
    int blocks = (int)((total + 255) / 256);
    if (blocks > 148 * 8) blocks = 148 * 8;
    silu_mul_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(gu),
                                            reinterpret_cast<__nv_bfloat16*>(act), M, I);
    return cudaGetLastError();
}

}  // namespace isd
