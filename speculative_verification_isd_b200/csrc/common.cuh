// Shared device helpers for the ISD kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/isd.h"
#include "plan.h"

#define ISD_DEVINL __device__ __forceinline__

namespace isd {

// Programmatic dependent launch: wait until the preceding kernel of the
// stream has completed and its memory is visible (a no-op for a kernel
// launched without the attribute); allow the next kernel to be scheduled.
ISD_DEVINL void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
ISD_DEVINL void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }


ISD_DEVINL void raise_flag(int32_t* err_flag, int32_t bit) {
    if (err_flag) atomicOr(err_flag, bit);
}

ISD_DEVINL uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous global->shared copy; src_bytes == 0 zero-fills.
ISD_DEVINL void cp_async16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
ISD_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
ISD_DEVINL void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

ISD_DEVINL void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
ISD_DEVINL void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, fp32 accumulate.
ISD_DEVINL void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

ISD_DEVINL uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Streaming 16-byte load that does not allocate in L1.
ISD_DEVINL float4 ld_stream_f4(const float* p) {
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];\n"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

// Running (max, sum exp(z - max), argmax) over a sequence of logits.
struct RowStat {
    float m;
    float s;
    int idx;
};

ISD_DEVINL RowStat rowstat_empty() { return RowStat{-INFINITY, 0.f, 0x7fffffff}; }

// Fold one element with a larger index than any already folded.
ISD_DEVINL void rowstat_push(RowStat& a, float z, int i) {
    if (z > a.m) {
        a.s = a.s * __expf(a.m - z) + 1.f;
        a.m = z;
        a.idx = i;
    } else {
        a.s += __expf(z - a.m);
    }
}

// Merge two partial statistics; equal maxima keep the lower index.
ISD_DEVINL RowStat rowstat_merge(RowStat a, RowStat b) {
    if (b.s == 0.f) return a;
    if (a.s == 0.f) return b;
    const float M = fmaxf(a.m, b.m);
    RowStat r;
    r.m = M;
    r.s = a.s * __expf(a.m - M) + b.s * __expf(b.m - M);
    r.idx = (a.m > b.m) ? a.idx : (b.m > a.m) ? b.idx : min(a.idx, b.idx);
    return r;
}

ISD_DEVINL RowStat rowstat_shfl_xor(const RowStat& a, int lane_mask) {
    RowStat o;
    o.m = __shfl_xor_sync(0xffffffffu, a.m, lane_mask);
    o.s = __shfl_xor_sync(0xffffffffu, a.s, lane_mask);
    o.idx = __shfl_xor_sync(0xffffffffu, a.idx, lane_mask);
    return o;
}

// Block-wide merge in a fixed order; result valid in thread 0.
template <int THREADS>
ISD_DEVINL RowStat rowstat_block_reduce(RowStat a) {
    __shared__ RowStat warp_part[THREADS / 32];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a = rowstat_merge(a, rowstat_shfl_xor(a, off));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) warp_part[warp] = a;
    __syncthreads();
    if (warp == 0) {
        // the warp partials, merged by warp 0 in a shuffle tree
        a = lane < THREADS / 32 ? warp_part[lane] : rowstat_empty();
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) a = rowstat_merge(a, rowstat_shfl_xor(a, off));
    }
    __syncthreads();
    return a;
}


// Row statistics from n <= kMaxStatParts partials p[0..n), merged by
// one warp in a fixed order: lane l folds p[l], p[l + 32], ... in index order,
// then the lanes meet in a fixed shuffle tree and lane 0's result is
// broadcast.  Every caller (the LM head's merge kernel, the accept kernel)
// uses this one routine, so the merged statistics are bit-identical.
constexpr int kMaxPartsPerLane = kMaxStatParts / 32;
template <int BATCH = 4>
ISD_DEVINL RowStat warp_merge_partials(const float4* p, int n) {
    const int lane = threadIdx.x & 31;
    RowStat st = rowstat_empty();
    // loads in batches of BATCH per lane (more in flight, more registers);
    // the order of the merge does not depend on BATCH
    for (int u0 = 0; u0 < kMaxPartsPerLane && 32 * u0 < n; u0 += BATCH) {
        float4 v[BATCH];
#pragma unroll
        for (int u = 0; u < BATCH; ++u) {
            const int k = lane + 32 * (u0 + u);
            v[u] = k < n ? __ldcg(p + k) : make_float4(-INFINITY, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < BATCH; ++u) st = rowstat_merge(st, RowStat{v[u].x, v[u].y, __float_as_int(v[u].z)});
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) st = rowstat_merge(st, rowstat_shfl_xor(st, off));
    st.m = __shfl_sync(0xffffffffu, st.m, 0);
    st.s = __shfl_sync(0xffffffffu, st.s, 0);
    st.idx = __shfl_sync(0xffffffffu, st.idx, 0);
    return st;
}

}  // namespace isd
