// KV append (a1) and strict-causal GQA attention over the paged cache (a2):
// the general kernel, for the shapes the tensor-core kernel in
// attention_tc.cu does not take (D = 64, more than 64 query rows per kv head,
// pages that are not 8..128 tokens dividing 128).  launch_attention at the
// end of this file picks the kernel.
//
// Strict causal attention over clean and MASK slots alike is the first of the
// training changes on "I-DLM：扩散模型如何用“自省一致性”追上自回归模型质量"
// (section "三项关键训练创新", 严格因果掩码); the paged KV cache is the AR
// serving structure the same page reuses (section "推理：复用 AR 推理栈").
//
// Design (B200, memory-bound: ~28 flop per KV byte):
//  * one CTA per (request, KV head, split of the key range, row block); the
//    grp*Q query rows that share a KV head (28 for Qwen3-8B at N=4) are
//    processed together, so every KV byte is read from HBM once;
//  * keys stream through a 3-stage cp.async pipeline in 64-key tiles gathered
//    page by page; a per-split key -> cache-row table (one page lookup per
//    key) keeps the per-tile address work to a load and a multiply-add;
//  * warps are arranged as (16-row group) x (16 keys of the tile): every warp
//    owns 16 query rows, so its output accumulator is 64 registers and two
//    CTAs of 8 warps fit on an SM (the kernel is latency-bound: warps hide
//    each other's mma.sync dependency chains);
//  * S = Q K^T and O += P V on mma.sync m16n8k16 (bf16 in, fp32 accumulate),
//    online softmax in the log2 domain with a lazily moved reference maximum;
//  * warps merge in a fixed order; splits of one (request, head) are merged
//    by the CTA that draws the last ticket (no spinning, deterministic);
//  * block keys are read from k_new/v_new directly, and the CTA of the last
//    split writes them into the pages, so the append needs no ordering.
#include "common.cuh"
#include "plan.h"

namespace isd {

constexpr int kStages = 3;
constexpr int kKT = kAttnKeyTile;

struct AttnArgs {
    int B, N, Q, Hq, Hkv, grp, rows, P, num_pages, max_pages, split, n_rgb;
    float scale_log2;  // sm_scale * log2(e)
    const __nv_bfloat16* q;
    const __nv_bfloat16* k_new;
    const __nv_bfloat16* v_new;
    __nv_bfloat16* k_pool;
    __nv_bfloat16* v_pool;
    const int32_t* page_table;
    const int32_t* kv_len;
    const int32_t* n_clean;  // null: every one of the N first slots is active (c = N)
    int bidir;               // 1: every row sees the whole block (block-causal mask)
    __nv_bfloat16* out;
    char* part;
    size_t part_stride;
    int max_splits;
    int* ticket;
    int32_t* err_flag;
};

// smem byte offset of 16-byte chunk `c` of row `r` (rows of D bf16)
template <int D>
ISD_DEVINL uint32_t swz(int r, int c) {
    return (uint32_t)(r * D * 2 + ((c ^ (r & 7)) << 4));
}

// position of block slot s (-1 = inactive), c clean tokens
ISD_DEVINL int slot_pos(int s, int kv, int c, int N) {
    if (s < c) return kv + s;
    if (s < N) return -1;
    return kv + c + (s - N);
}

template <int D, int RG>
__global__ void __launch_bounds__(128 * RG, (RG <= 2 ? 2 : 1)) attention_kernel(const __grid_constant__ AttnArgs a) {
    constexpr int THREADS = 128 * RG;
    constexpr int ROWS = 16 * RG;  // query rows of this CTA
    constexpr int CH = D / 8;      // 16-byte chunks per row
    constexpr int NT = D / 8;      // n8 tiles of the output
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char* sQ = smem;
    unsigned char* sK = smem + ROWS * D * 2;
    unsigned char* sV = sK + kStages * kKT * D * 2;

    const int sp = blockIdx.x;
    const int g = blockIdx.y / a.n_rgb;
    const int rgb = blockIdx.y % a.n_rgb;
    const int b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rg = warp >> 2;          // 16-row group of this warp
    const int kw = (warp & 3) * 16;    // this warp's keys within a tile

    const int kv = a.kv_len[b];
    const int c = a.n_clean ? a.n_clean[b] : a.N;
    const bool bad_c = (c < 1 || c > a.N);
    // keys incl. the block: c clean slots, then the Q - N slots after them
    const long long want = bad_c ? 0 : (long long)kv + c + a.Q - a.N;
    const bool over = kv < 0 || (want + a.P - 1) / a.P > a.max_pages;
    // a request that cannot be served (bad n_clean, negative or over-capacity
    // length) is one empty split: its rows are written as zeros
    const int total = (bad_c || over) ? 0 : (int)want;
    const int ns = total > 0 ? (total + a.split - 1) / a.split : 1;
    if (sp >= ns) return;
    if (tid == 0 && sp == 0 && rgb == 0) {
        if (bad_c) raise_flag(a.err_flag, ISD_FLAG_NCLEAN_RANGE);
        else if (over) raise_flag(a.err_flag, ISD_FLAG_CAPACITY);
    }
    const int kbeg = sp * a.split;
    const int kend = min(total, kbeg + a.split);
    const int32_t* ptab = a.page_table + (size_t)b * a.max_pages;
    const size_t row_stride = (size_t)a.Hkv * D;  // elements between consecutive positions

    // ---- a1: the last split's CTA appends the block's K/V rows to the pages
    if (sp == ns - 1 && rgb == 0 && total > 0) {
        const int nblk = c + a.Q - a.N;
        for (int i = tid; i < nblk * CH; i += THREADS) {
            const int r = i / CH, cc = i % CH;
            const int t = kv + r;
            const int slot = r < c ? r : a.N + (r - c);
            const int page = ptab[t / a.P];
            if (page < 0 || page >= a.num_pages) {
                raise_flag(a.err_flag, ISD_FLAG_PAGE_OOB);
                continue;
            }
            const size_t dst = ((size_t)page * a.P + t % a.P) * row_stride + (size_t)g * D + cc * 8;
            const size_t src = (((size_t)b * a.Q + slot) * a.Hkv + g) * D + cc * 8;
            *reinterpret_cast<uint4*>(a.k_pool + dst) = *reinterpret_cast<const uint4*>(a.k_new + src);
            *reinterpret_cast<uint4*>(a.v_pool + dst) = *reinterpret_cast<const uint4*>(a.v_new + src);
        }
    }

    // ---- query rows of this CTA -> smem (zero rows for padding)
    const int row0 = rgb * ROWS;
    for (int i = tid; i < ROWS * CH; i += THREADS) {
        const int r = i / CH, cc = i % CH;
        const int rr = row0 + r;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (rr < a.rows) {
            const int hh = rr / a.Q, s = rr % a.Q;
            const int h = g * a.grp + hh;
            v = *reinterpret_cast<const uint4*>(a.q + (((size_t)b * a.Q + s) * a.Hq + h) * D + cc * 8);
        }
        *reinterpret_cast<uint4*>(sQ + swz<D>(r, cc)) = v;
    }

    // positions of the 2 rows this thread holds in the S/O fragments
    int rpos[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int rr = row0 + rg * 16 + i * 8 + (lane >> 2);
        rpos[i] = (rr < a.rows && total > 0) ? slot_pos(rr % a.Q, kv, c, a.N) : -1;
        if (a.bidir && rpos[i] >= 0) rpos[i] = total - 1;
    }

    // ---- key -> cache-row table of this split (one page lookup per key):
    //   >= 0      : pool row page*P + t%P (prefix keys)
    //   -(slot+1) : the block's own slot `slot` in k_new / v_new
    //   kNoKey    : nothing to load (bad page id); the chunk is zero-filled
    constexpr int kNoKey = INT_MIN;
    int* s_rows = reinterpret_cast<int*>(sV + kStages * kKT * D * 2);
    const int nkeys = kend - kbeg;
    for (int k = tid; k < nkeys; k += THREADS) {
        const int t = kbeg + k;
        int row;
        if (t < kv) {
            const int page = ptab[t / a.P];
            if (page >= 0 && page < a.num_pages) {
                row = page * a.P + t % a.P;
            } else {
                raise_flag(a.err_flag, ISD_FLAG_PAGE_OOB);
                row = kNoKey;
            }
        } else {
            const int r = t - kv;
            row = -((r < c ? r : a.N + (r - c)) + 1);
        }
        s_rows[k] = row;
    }
    __syncthreads();

    // ---- tile loader: each thread always copies chunk `cc` of keys
    //      kr0 + j*KPP, so its swizzled smem offset is a per-thread constant
    constexpr int KPP = THREADS / CH;  // keys per pass (a multiple of 8)
    constexpr int PASSES = kKT / KPP;
    static_assert(KPP % 8 == 0 && kKT % KPP == 0, "constant swizzle needs 8-key passes");
    const int cc = tid % CH, kr0 = tid / CH;
    const size_t pool_col = (size_t)g * D + cc * 8;
    const __nv_bfloat16* knew_b = a.k_new + ((size_t)b * a.Q * a.Hkv + g) * D + cc * 8;
    const __nv_bfloat16* vnew_b = a.v_new + ((size_t)b * a.Q * a.Hkv + g) * D + cc * 8;
    const size_t slot_stride = (size_t)a.Hkv * D;
    const uint32_t dst0 = (uint32_t)(kr0 * D * 2 + ((cc ^ (kr0 & 7)) << 4));
    auto load_tile = [&](int stage, int tile) {
        const uint32_t dk = smem_u32(sK + stage * kKT * D * 2) + dst0;
        const uint32_t dv = smem_u32(sV + stage * kKT * D * 2) + dst0;
#pragma unroll
        for (int j = 0; j < PASSES; ++j) {
            const int k = tile * kKT + kr0 + j * KPP;
            const int row = k < nkeys ? s_rows[k] : kNoKey;
            const __nv_bfloat16* sk = a.k_new;
            const __nv_bfloat16* sv = a.v_new;
            int bytes = 16;
            if (row >= 0) {
                sk = a.k_pool + (size_t)row * row_stride + pool_col;
                sv = a.v_pool + (size_t)row * row_stride + pool_col;
            } else if (row != kNoKey) {
                sk = knew_b + (size_t)(-row - 1) * slot_stride;
                sv = vnew_b + (size_t)(-row - 1) * slot_stride;
            } else {
                bytes = 0;
            }
            cp_async16(dk + j * KPP * D * 2, sk, bytes);
            cp_async16(dv + j * KPP * D * 2, sv, bytes);
        }
    };

    float o[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
    // running reference max (log2 domain) and running sum of each row
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    // Keys below mask_from are cached prefix keys of a live split: visible to
    // every active row, so their tiles need no masking.
    const int mask_from = min(kv, kend);
    // The reference max only moves when a row's max exceeds it by more than
    // 2^8: probabilities are then at most 256 (exact in fp32, same relative
    // precision in bf16) and the O rescale is skipped almost always.  The
    // result is independent of the reference after the final normalisation.
    constexpr float kRescaleThreshold = 8.f;

    const int n_tiles = (nkeys + kKT - 1) / kKT;
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        if (s < n_tiles) load_tile(s, s);
        cp_async_commit();
    }
    const int l7 = lane & 7, j8 = lane >> 3;
    const uint32_t q_row = smem_u32(sQ) + (uint32_t)((rg * 16 + (j8 & 1) * 8 + l7) * D * 2);
    for (int it = 0; it < n_tiles; ++it) {
        cp_async_wait<kStages - 2>();
        __syncthreads();
        {
            const int nxt = it + kStages - 1;
            if (nxt < n_tiles) load_tile(nxt % kStages, nxt);
            cp_async_commit();
        }
        const int stage = it % kStages;
        const uint32_t k_base = smem_u32(sK + stage * kKT * D * 2);
        const uint32_t v_base = smem_u32(sV + stage * kKT * D * 2);
        const int k0 = kbeg + it * kKT + kw;  // first key of this warp
        if (k0 >= kend) continue;             // warp has no keys in this tile

        // S = Q K^T  (16 rows x 16 keys); rows and keys of every ldmatrix
        // start at multiples of 8, so the swizzle XOR is lane & 7
        float s[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
        const uint32_t k_row = k_base + (uint32_t)((kw + (j8 >> 1) * 8 + l7) * D * 2);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t kb[4], qa[4];
            ldmatrix_x4(kb, k_row + (uint32_t)(((kk * 2 + (j8 & 1)) ^ l7) << 4));
            ldmatrix_x4(qa, q_row + (uint32_t)(((kk * 2 + (j8 >> 1)) ^ l7) << 4));
            mma_bf16_16816(s[0], qa, kb[0], kb[1]);
            mma_bf16_16816(s[1], qa, kb[2], kb[3]);
        }
        // mask (boundary tiles only) + online softmax in the log2 domain
        if (k0 + 16 > mask_from) {
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int key = k0 + nt * 8 + (lane & 3) * 2 + e;
                        if (key >= kend || key > rpos[i]) s[nt][i * 2 + e] = -INFINITY;
                    }
        }
        float alpha[2];
        bool moved = false;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float mx = fmaxf(fmaxf(s[0][i * 2], s[0][i * 2 + 1]), fmaxf(s[1][i * 2], s[1][i * 2 + 1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            mx *= a.scale_log2;
            alpha[i] = 1.f;
            if (mx > m_run[i] + kRescaleThreshold || (m_run[i] == -INFINITY && mx > -INFINITY)) {
                alpha[i] = exp2f(m_run[i] - mx);
                m_run[i] = mx;
                moved = true;
            }
            const float m_use = (m_run[i] == -INFINITY) ? 0.f : m_run[i];
            float rs = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float p = exp2f(fmaf(s[nt][i * 2 + e], a.scale_log2, -m_use));
                    s[nt][i * 2 + e] = p;
                    rs += p;
                }
            rs += __shfl_xor_sync(0xffffffffu, rs, 1);
            rs += __shfl_xor_sync(0xffffffffu, rs, 2);
            l_run[i] = l_run[i] * alpha[i] + rs;
        }
        if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                o[nt][0] *= alpha[0];
                o[nt][1] *= alpha[0];
                o[nt][2] *= alpha[1];
                o[nt][3] *= alpha[1];
            }
        }
        // O += P V  (P: 16 rows x 16 keys as the A operand, from the S fragments)
        uint32_t pa[4];
        pa[0] = pack_bf16(s[0][0], s[0][1]);
        pa[1] = pack_bf16(s[0][2], s[0][3]);
        pa[2] = pack_bf16(s[1][0], s[1][1]);
        pa[3] = pack_bf16(s[1][2], s[1][3]);
        const uint32_t v_row = v_base + (uint32_t)((kw + (j8 & 1) * 8 + l7) * D * 2);
#pragma unroll
        for (int dn = 0; dn < NT; dn += 2) {
            uint32_t vb[4];
            ldmatrix_x4_trans(vb, v_row + (uint32_t)(((dn + (j8 >> 1)) ^ l7) << 4));
            mma_bf16_16816(o[dn], pa, vb[0], vb[1]);
            mma_bf16_16816(o[dn + 1], pa, vb[2], vb[3]);
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- merge the 4 warps of each row group in a fixed order
    float* red = reinterpret_cast<float*>(sK);   // pipeline buffers are free now
    float* sm = red;                              // [warps][16] running max
    float* sl = red + THREADS / 32 * 16;          // [warps][16] running sum
    float* obuf = red + 2 * (THREADS / 32) * 16;  // [rg][2][NT*4][32]
    const int wig = warp & 3;  // warp index within its row group
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        // inactive / padding rows were not masked in prefix tiles: drop them
        if (rpos[i] < 0) {
            m_run[i] = -INFINITY;
            l_run[i] = 0.f;
        }
    }
    if ((lane & 3) == 0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = i * 8 + (lane >> 2);
            sm[warp * 16 + r] = m_run[i];
            sl[warp * 16 + r] = l_run[i];
        }
    }
    __syncthreads();
    float m_fin[2], l_fin[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = i * 8 + (lane >> 2);
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, sm[(rg * 4 + w) * 16 + r]);
        const float Mu = (M == -INFINITY) ? 0.f : M;
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int ww = (rg * 4 + w) * 16 + r;
            L += sl[ww] * exp2f(sm[ww] - Mu);
        }
        const float f = exp2f(m_run[i] - Mu);
        m_fin[i] = M;
        l_fin[i] = L;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            o[nt][i * 2] *= f;
            o[nt][i * 2 + 1] *= f;
        }
    }
    constexpr int buf_elems = NT * 4 * 32;
    float* my_buf = obuf + (size_t)(rg * 2) * buf_elems;  // two buffers per row group
    auto store_o = [&](float* buf) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) buf[(nt * 4 + e) * 32 + lane] = o[nt][e];
    };
    auto add_o = [&](const float* buf) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[nt][e] += buf[(nt * 4 + e) * 32 + lane];
    };
    __syncthreads();
    if (wig >= 2) store_o(my_buf + (wig - 2) * buf_elems);
    __syncthreads();
    if (wig < 2) add_o(my_buf + wig * buf_elems);
    __syncthreads();
    if (wig == 1) store_o(my_buf);
    __syncthreads();
    if (wig == 0) add_o(my_buf);

    // ---- write: direct output (single split) or a partial + ticket combine
    const size_t unit = ((size_t)b * a.Hkv + g) * a.n_rgb + rgb;
    if (ns == 1) {
        if (wig == 0) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int rr = row0 + rg * 16 + i * 8 + (lane >> 2);
                if (rr >= a.rows) continue;
                const int hh = rr / a.Q, s = rr % a.Q;
                const int h = g * a.grp + hh;
                const float inv = l_fin[i] > 0.f ? 1.f / l_fin[i] : 0.f;
                __nv_bfloat16* dst = a.out + ((size_t)b * a.Q + s) * a.Hq * D + (size_t)h * D;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int col = nt * 8 + (lane & 3) * 2;
                    *reinterpret_cast<__nv_bfloat162*>(dst + col) =
                        __floats2bfloat162_rn(o[nt][i * 2] * inv, o[nt][i * 2 + 1] * inv);
                }
            }
        }
        return;
    }
    // partial: m[ROWS], l[ROWS], O[ROWS][D] (fp32, O scaled to m)
    char* pbase = a.part + (unit * a.max_splits + sp) * a.part_stride;
    float* pm = reinterpret_cast<float*>(pbase);
    float* pl = pm + ROWS;
    float* po = pl + ROWS;
    if (wig == 0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = rg * 16 + i * 8 + (lane >> 2);
            if ((lane & 3) == 0) {
                pm[r] = m_fin[i];
                pl[r] = l_fin[i];
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int col = nt * 8 + (lane & 3) * 2;
                *reinterpret_cast<float2*>(po + (size_t)r * D + col) =
                    make_float2(o[nt][i * 2], o[nt][i * 2 + 1]);
            }
        }
    }
    __threadfence();
    __syncthreads();
    __shared__ int s_last;
    if (tid == 0) s_last = (atomicAdd(&a.ticket[unit], 1) == ns - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // combine all splits in order 0..ns-1
    const char* ubase = a.part + unit * a.max_splits * a.part_stride;
    for (int i = tid; i < ROWS * (D / 2); i += THREADS) {
        const int r = i / (D / 2), col = (i % (D / 2)) * 2;
        const int rr = row0 + r;
        if (rr >= a.rows) continue;
        float M = -INFINITY;
        for (int k = 0; k < ns; ++k)
            M = fmaxf(M, __ldcg(reinterpret_cast<const float*>(ubase + k * a.part_stride) + r));
        const float Mu = (M == -INFINITY) ? 0.f : M;
        float L = 0.f, o0 = 0.f, o1 = 0.f;
        for (int k = 0; k < ns; ++k) {
            const float* km = reinterpret_cast<const float*>(ubase + k * a.part_stride);
            const float f = exp2f(__ldcg(km + r) - Mu);
            L += __ldcg(km + ROWS + r) * f;
            const float2 ov = __ldcg(reinterpret_cast<const float2*>(km + 2 * ROWS + (size_t)r * D + col));
            o0 += ov.x * f;
            o1 += ov.y * f;
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        const int hh = rr / a.Q, s = rr % a.Q;
        const int h = g * a.grp + hh;
        __nv_bfloat16* dst = a.out + ((size_t)b * a.Q + s) * a.Hq * D + (size_t)h * D + col;
        *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(o0 * inv, o1 * inv);
    }
    if (tid == 0) a.ticket[unit] = 0;
}

template <int D, int RG>
static size_t attn_smem_bytes(int split) {
    // Q rows + K/V pipeline stages + the split's key -> row table
    return (size_t)16 * RG * D * 2 + (size_t)2 * kStages * kKT * D * 2 + (size_t)split * 4;
}

template <int D, int RG>
static cudaError_t launch_attention_t(const AttnArgs& a, dim3 grid, cudaStream_t st) {
    static unsigned long long configured = 0;  // bit per device: attribute set
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!(configured >> dev & 1ull)) {
        cudaError_t e = cudaFuncSetAttribute(attention_kernel<D, RG>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)attn_smem_bytes<D, RG>(kAttnMaxSplit));
        if (e != cudaSuccess) return e;
        configured |= 1ull << dev;
    }
    attention_kernel<D, RG><<<grid, 128 * RG, attn_smem_bytes<D, RG>(a.split), st>>>(a);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_attention_d(int rg, const AttnArgs& a, dim3 grid, cudaStream_t st) {
    if (rg == 1) return launch_attention_t<D, 1>(a, grid, st);
    if (rg == 2) return launch_attention_t<D, 2>(a, grid, st);
    return launch_attention_t<D, 4>(a, grid, st);
}

cudaError_t launch_attention_tc(const Plan& p, const isd_dims* d, const uint16_t* q,
                                const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_pool,
                                uint16_t* v_pool, const int32_t* page_table, const int32_t* kv_len,
                                const int32_t* n_clean, uint16_t* out, void* ws, int32_t* err_flag,
                                cudaStream_t st, int* clear_extra, int* clear_range, int clear_count,
                                bool pdl, bool bidir, bool* handled);

// The tensor-core kernel (attention_tc.cu) where the shape fits it, else the
// general mma.sync kernel above.  Either way the attention counters in the
// workspace are cleared on the stream first, and so are the B counters at
// clear_extra (2 B + 1: the accept kernel's tickets, states and decided count) and the
// clear_count counters at clear_range when not null.
// pdl: launched as part of the whole step (programmatic dependent launch).
cudaError_t launch_attention(const Plan& p, const isd_dims* d, const uint16_t* q,
                             const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_pool,
                             uint16_t* v_pool, const int32_t* page_table, const int32_t* kv_len,
                             const int32_t* n_clean, uint16_t* out, void* ws, int32_t* err_flag,
                             cudaStream_t st, int* clear_extra, int* clear_range, int clear_count,
                             bool pdl, bool bidir) {
    bool handled = false;
    const cudaError_t te = launch_attention_tc(p, d, q, k_new, v_new, k_pool, v_pool, page_table,
                                               kv_len, n_clean, out, ws, err_flag, st, clear_extra,
                                               clear_range, clear_count, pdl, bidir, &handled);
    if (handled || te != cudaSuccess) return te;
    cudaError_t me = cudaMemsetAsync(static_cast<char*>(ws) + p.off_attn_ticket, 0,
                                     (size_t)d->B * d->Hkv * p.attn_rgb * 4, st);
    if (me == cudaSuccess && clear_extra) me = cudaMemsetAsync(clear_extra, 0, (size_t)d->B * 2 * 4 + 4, st);
    if (me == cudaSuccess && clear_range && clear_count > 0)
        me = cudaMemsetAsync(clear_range, 0, (size_t)clear_count * 4, st);
    if (me != cudaSuccess) return me;
    char* w = static_cast<char*>(ws);
    AttnArgs a;
    a.B = d->B;
    a.N = d->N;
    a.Q = p.Q;
    a.Hq = d->Hq;
    a.Hkv = d->Hkv;
    a.grp = p.grp;
    a.rows = p.rows;
    a.P = d->page_size;
    a.num_pages = d->num_pages;
    a.max_pages = d->max_pages_per_req;
    a.split = p.attn_split;
    a.n_rgb = p.attn_rgb;
    a.scale_log2 = d->sm_scale * 1.4426950408889634f;
    a.q = reinterpret_cast<const __nv_bfloat16*>(q);
    a.k_new = reinterpret_cast<const __nv_bfloat16*>(k_new);
    a.v_new = reinterpret_cast<const __nv_bfloat16*>(v_new);
    a.k_pool = reinterpret_cast<__nv_bfloat16*>(k_pool);
    a.v_pool = reinterpret_cast<__nv_bfloat16*>(v_pool);
    a.page_table = page_table;
    a.kv_len = kv_len;
    a.n_clean = n_clean;
    a.bidir = bidir ? 1 : 0;
    a.out = reinterpret_cast<__nv_bfloat16*>(out);
    a.part = w + p.off_attn_part;
    a.part_stride = p.attn_part_stride;
    a.max_splits = p.attn_max_splits;
    a.ticket = reinterpret_cast<int*>(w + p.off_attn_ticket);
    a.err_flag = err_flag;
    dim3 grid(p.attn_max_splits, d->Hkv * p.attn_rgb, d->B);
    if (d->D == 128) return launch_attention_d<128>(p.attn_rg, a, grid, st);
    return launch_attention_d<64>(p.attn_rg, a, grid, st);
}

}  // namespace isd
