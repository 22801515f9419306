// HBM-bound kernels of the owner step: Nesterov momentum with the Frobenius
// partial sums and the short-side-first layout of X, the per-matrix norm
// finalisation, the ns_steps = 0 parameter write, and AdamW over the packed
// tail.  Method passages: arxivlens summary page of "MatrixFSDP", Abstract
// (momentum-smoothed Muon update on the owner; tail on AdamW).
#include "internal.h"
#include "master.cuh"

#include <cuda_bf16.h>
#include <cstdint>

namespace mfsdp {
namespace {

__device__ __forceinline__ void record_status(int32_t* status, int32_t code) {
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float load_elem(const void* p, int64_t i, int bf16) {
    return bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i])
                : static_cast<const float*>(p)[i];
}

// four consecutive elements at p[i..i+3]; i % 4 == 0 and the base aligned
__device__ __forceinline__ float4 load4(const void* p, int64_t i, int bf16) {
    if (bf16) {
        uint2 raw = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(p) + i);
        __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
        __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
        float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
        return make_float4(a.x, a.y, b.x, b.y);
    }
    return *reinterpret_cast<const float4*>(static_cast<const float*>(p) + i);
}

__device__ __forceinline__ void store4_bf16(__nv_bfloat16* p, int64_t i, float4 v) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 raw;
    raw.x = *reinterpret_cast<uint32_t*>(&lo);
    raw.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p + i) = raw;
}

// bf16-mode master of X (master.cuh) at i..i+3, i % 4 == 0: hi and lo parts
__device__ __forceinline__ void store4_master(__nv_bfloat16* xb, __nv_bfloat16* xlo, int64_t i, float4 v) {
    uint16_t h0, h1, h2, h3, l0, l1, l2, l3;
    master_split(v.x, h0, l0);
    master_split(v.y, h1, l1);
    master_split(v.z, h2, l2);
    master_split(v.w, h3, l3);
    *reinterpret_cast<uint2*>(xb + i) = make_uint2(static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16),
                                                   static_cast<uint32_t>(h2) | (static_cast<uint32_t>(h3) << 16));
    *reinterpret_cast<uint2*>(xlo + i) = make_uint2(static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16),
                                                    static_cast<uint32_t>(l2) | (static_cast<uint32_t>(l3) << 16));
}

__device__ __forceinline__ void store1_master(__nv_bfloat16* xb, __nv_bfloat16* xlo, int64_t i, float v) {
    uint16_t h, l;
    master_split(v, h, l);
    xb[i] = __ushort_as_bfloat16(h);
    xlo[i] = __ushort_as_bfloat16(l);
}

__device__ __forceinline__ float4 load4_master(const __nv_bfloat16* xb, const __nv_bfloat16* xlo, int64_t i) {
    const uint2 h = *reinterpret_cast<const uint2*>(xb + i);
    const uint2 l = *reinterpret_cast<const uint2*>(xlo + i);
    return make_float4(master_value(static_cast<uint16_t>(h.x & 0xFFFFu), static_cast<uint16_t>(l.x & 0xFFFFu)),
                       master_value(static_cast<uint16_t>(h.x >> 16), static_cast<uint16_t>(l.x >> 16)),
                       master_value(static_cast<uint16_t>(h.y & 0xFFFFu), static_cast<uint16_t>(l.y & 0xFFFFu)),
                       master_value(static_cast<uint16_t>(h.y >> 16), static_cast<uint16_t>(l.y >> 16)));
}

__device__ __forceinline__ float load1_master(const __nv_bfloat16* xb, const __nv_bfloat16* xlo, int64_t i) {
    return master_value(__bfloat16_as_ushort(xb[i]), __bfloat16_as_ushort(xlo[i]));
}

// eight consecutive elements at p[i..i+7] as floats; i % 8 == 0 and p + i 16-byte aligned
__device__ __forceinline__ void load8(const void* p, int64_t i, int bf16, float (&v)[8]) {
    if (bf16) {
        const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p) + i));
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        #pragma unroll
        for (int k = 0; k < 4; ++k) {
            v[2 * k] = __uint_as_float(w[k] << 16);
            v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
        }
    } else {
        const float4 a = __ldcs(reinterpret_cast<const float4*>(static_cast<const float*>(p) + i));
        const float4 b = __ldcs(reinterpret_cast<const float4*>(static_cast<const float*>(p) + i) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

// bf16-mode master of X (master.cuh) at i..i+7, i % 8 == 0: one 16-byte store of each part
__device__ __forceinline__ void store8_master(__nv_bfloat16* xb, __nv_bfloat16* xlo, int64_t i, const float (&v)[8]) {
    uint32_t h[4], l[4];
    #pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint16_t h0, l0, h1, l1;
        master_split(v[2 * k], h0, l0);
        master_split(v[2 * k + 1], h1, l1);
        h[k] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
        l[k] = static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
    }
    *reinterpret_cast<uint4*>(xb + i) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(xlo + i) = make_uint4(l[0], l[1], l[2], l[3]);
}

// index of the matrix owning tile group `grp` (largest i with mom_grp0 <= grp)
__device__ __forceinline__ int find_matrix(const MatDev* mats, int nmats, int grp) {
    int lo = 0, hi = nmats - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (mats[mid].mom_grp0 <= grp) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// deterministic block sum (fixed shuffle tree, fixed warp order)
template <typename T>
__device__ __forceinline__ T block_sum(T v, T* smem) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) smem[warp] = v;
    __syncthreads();
    T r = 0;
    if (threadIdx.x == 0) {
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r += smem[w];
    }
    return r;  // valid in thread 0
}

// Momentum over one flat group of an untransposed matrix: elements [e0, e0 + kFlatGroup)
// of M (and of X, whose leading dimension is cols), in runs of 8 per thread, U runs
// loaded before any arithmetic.  Returns this thread's sum of M^2.  GB: the gradient
// is bf16 (else fp32; PARTS reads the owner-segment parts of either dtype).  U = 4 with
// packed bf16 gradients; U = 2 otherwise.
template <int U, bool PARTS, bool GB>
__device__ __forceinline__ float momentum_flat(const MatDev& md, const StepScalars& sc, float* __restrict__ bufp,
                                               const void* gradp, const void* const* parts, int nparts, int64_t e0,
                                               int64_t n) {
    const float beta = sc.beta, omb = 1.0f - sc.beta;
    const int gbf = md.grad_bf16;
    float* __restrict__ xf = md.xf[0];
    __nv_bfloat16* __restrict__ xb = md.xb[0];
    __nv_bfloat16* __restrict__ xl = md.xlo[0];
    float sumsq = 0.f;
    #pragma unroll 1
    for (int c0 = 0; c0 < kFlatGroup / 8; c0 += U * 256) {
        float4 bq[U][2];
        uint4 gq[U][2];
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = e0 + 8 * (int64_t)(c0 + u * 256 + threadIdx.x);
            if (i >= n) continue;
            bq[u][0] = __ldcs(reinterpret_cast<const float4*>(bufp + i));
            bq[u][1] = __ldcs(reinterpret_cast<const float4*>(bufp + i) + 1);
            if (!PARTS) {
                if (GB) {
                    gq[u][0] = __ldcs(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(gradp) + i));
                } else {
                    gq[u][0] = __ldcs(reinterpret_cast<const uint4*>(static_cast<const float*>(gradp) + i));
                    gq[u][1] = __ldcs(reinterpret_cast<const uint4*>(static_cast<const float*>(gradp) + i) + 1);
                }
            }
        }
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = e0 + 8 * (int64_t)(c0 + u * 256 + threadIdx.x);
            if (i >= n) continue;
            float gv[8];
            if (!PARTS) {
                if (GB) {
                    const uint32_t w[4] = {gq[u][0].x, gq[u][0].y, gq[u][0].z, gq[u][0].w};
                    #pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        gv[2 * k] = __uint_as_float(w[k] << 16);
                        gv[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
                    }
                } else {
                    const uint32_t w[8] = {gq[u][0].x, gq[u][0].y, gq[u][0].z, gq[u][0].w,
                                           gq[u][1].x, gq[u][1].y, gq[u][1].z, gq[u][1].w};
                    #pragma unroll
                    for (int k = 0; k < 8; ++k) gv[k] = __uint_as_float(w[k]);
                }
            } else {
                // the owner's gradient: contributions summed in rank order, in fp32
                load8(parts[0], i, gbf, gv);
                for (int r = 1; r < nparts; ++r) {
                    float q[8];
                    load8(parts[r], i, gbf, q);
                    #pragma unroll
                    for (int k = 0; k < 8; ++k) gv[k] += q[k];
                }
            }
            const float bin[8] = {bq[u][0].x, bq[u][0].y, bq[u][0].z, bq[u][0].w,
                                  bq[u][1].x, bq[u][1].y, bq[u][1].z, bq[u][1].w};
            float bo[8], m[8];
            #pragma unroll
            for (int k = 0; k < 8; ++k) {
                bo[k] = beta * bin[k] + omb * gv[k];
                m[k] = sc.nesterov ? omb * gv[k] + beta * bo[k] : bo[k];
                sumsq += m[k] * m[k];
            }
            __stcs(reinterpret_cast<float4*>(bufp + i), make_float4(bo[0], bo[1], bo[2], bo[3]));
            __stcs(reinterpret_cast<float4*>(bufp + i) + 1, make_float4(bo[4], bo[5], bo[6], bo[7]));
            if (sc.bf16_mode) {
                store8_master(xb, xl, i, m);
            } else {
                *reinterpret_cast<float4*>(xf + i) = make_float4(m[0], m[1], m[2], m[3]);
                *reinterpret_cast<float4*>(xf + i + 4) = make_float4(m[4], m[5], m[6], m[7]);
            }
        }
    }
    return sumsq;
}

// ---------------------------------------------------------------------------
// K1: one 64 x 64 tile of M per block of 256 threads.
//   buf <- beta buf + (1-beta) G ;  M <- (1-beta) G + beta buf  (or M <- buf)
// writes buf and X = M, or M^T when rows > cols (bf16 mode: hi and lo parts,
// the hi part being the first GEMM operand; fp32 mode: fp32).  A block handles
// kMomGroup tiles of one matrix and writes the group's sum of M^2 to
// partials[group].  Untransposed tiles run without block barriers; transposed
// ones alternate between two staging tiles, one barrier each.
// ---------------------------------------------------------------------------
template <bool PARTS>
__global__ void __launch_bounds__(256, 4)
momentum_kernel(const MatDev* __restrict__ mats, int nmats, int grp_base, StepScalars sc,
                float* __restrict__ partials, int32_t* status) {
    __shared__ float tileM2[2][kMomTile][kMomTile + 1];
    __shared__ float red[8];
    const int grp = grp_base + blockIdx.x;
    const int mi = find_matrix(mats, nmats, grp);
    const MatDev& md = mats[mi];
    const int64_t rows = md.rows, cols = md.cols;
    const int64_t tiles_m = (rows + kMomTile - 1) / kMomTile;
    // fields used inside the tile loop, read once (the loop's stores could otherwise force reloads)
    float* __restrict__ bufp = md.buf;
    const void* gradp = md.grad;
    const void* const* parts = md.gparts;   // owner-segment contributions (nparts > 0)
    const int nparts = md.nparts;
    const int mom_vec = md.mom_vec, tiles_n = md.mom_tiles_n, grp0 = md.mom_grp0;
    const int64_t ntiles = tiles_m * md.mom_tiles_n;
    if (grp < grp0) {  // cannot happen with a host-built table
        record_status(status, -7);
        return;
    }
    float sumsq = 0.f;
    for (int k = 0; k < kMomGroup; ++k) {
    const int local = (grp - grp0) * kMomGroup + k;
    if (local >= ntiles) break;      // block-uniform
    float (*tileM)[kMomTile + 1] = tileM2[k & 1];
    const int ti = local / tiles_n, tj = local % tiles_n;
    const int64_t i0 = (int64_t)ti * kMomTile, j0 = (int64_t)tj * kMomTile;
    const bool full = (i0 + kMomTile <= rows) && (j0 + kMomTile <= cols);
    const float beta = sc.beta, omb = 1.0f - sc.beta;
    const int tr = md.tr, gbf = md.grad_bf16, bf16_mode = sc.bf16_mode;
    float* __restrict__ xf = md.xf[0];          // fp32 mode
    __nv_bfloat16* __restrict__ xb = md.xb[0];  // bf16 mode: hi part ...
    __nv_bfloat16* __restrict__ xl = md.xlo[0]; // ... and lo part
    const int64_t ldx = md.ldx;

    if (full && mom_vec) {
        // the next tile's momentum and gradient lines into L2 (one thread per 128-byte line)
        if (!PARTS && k + 1 < kMomGroup && local + 1 < ntiles) {
            const int tin = (local + 1) / tiles_n, tjn = (local + 1) % tiles_n;
            const int64_t in0 = (int64_t)tin * kMomTile, jn0 = (int64_t)tjn * kMomTile;
            if (in0 + kMomTile <= rows && jn0 + kMomTile <= cols) {
                #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int v = e * 256 + threadIdx.x;
                    const int64_t pidx = (in0 + (v >> 4)) * cols + jn0 + (v & 15) * 4;
                    if ((v & 7) == 0) asm volatile("prefetch.global.L2 [%0];" ::"l"(bufp + pidx));
                    if ((v & (gbf ? 15 : 7)) == 0)
                        asm volatile("prefetch.global.L2 [%0];"
                                     ::"l"(gbf ? static_cast<const void*>(static_cast<const __nv_bfloat16*>(gradp) + pidx)
                                               : static_cast<const void*>(static_cast<const float*>(gradp) + pidx)));
                }
            }
        }
        // all eight 16-byte loads of this thread are issued before any store
        float4 b[4], g[4];
        int64_t idx[4];
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int v = e * 256 + threadIdx.x;
            idx[e] = (i0 + (v >> 4)) * cols + j0 + (v & 15) * 4;
            b[e] = __ldcs(reinterpret_cast<const float4*>(bufp + idx[e]));
            if (!PARTS) {
                g[e] = load4(gradp, idx[e], gbf);
            } else {
                // the owner's gradient: contributions summed in rank order, in fp32
                g[e] = load4(parts[0], idx[e], gbf);
                for (int r = 1; r < nparts; ++r) {
                    const float4 q = load4(parts[r], idx[e], gbf);
                    g[e].x += q.x; g[e].y += q.y; g[e].z += q.z; g[e].w += q.w;
                }
            }
        }
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int v = e * 256 + threadIdx.x;
            const int row = v >> 4, col = (v & 15) * 4;
            float4 bb = b[e];
            const float4 gg = g[e];
            float4 m;
            bb.x = beta * bb.x + omb * gg.x;  bb.y = beta * bb.y + omb * gg.y;
            bb.z = beta * bb.z + omb * gg.z;  bb.w = beta * bb.w + omb * gg.w;
            if (sc.nesterov) {
                m.x = omb * gg.x + beta * bb.x;  m.y = omb * gg.y + beta * bb.y;
                m.z = omb * gg.z + beta * bb.z;  m.w = omb * gg.w + beta * bb.w;
            } else {
                m = bb;
            }
            __stcs(reinterpret_cast<float4*>(bufp + idx[e]), bb);
            sumsq += m.x * m.x + m.y * m.y + m.z * m.z + m.w * m.w;
            if (!tr) {
                const int64_t xi = (i0 + row) * ldx + j0 + col;
                if (bf16_mode) store4_master(xb, xl, xi, m);
                else *reinterpret_cast<float4*>(xf + xi) = m;
            } else {
                tileM[row][col] = m.x; tileM[row][col + 1] = m.y;
                tileM[row][col + 2] = m.z; tileM[row][col + 3] = m.w;
            }
        }
    } else {
        for (int e = 0; e < 16; ++e) {
            const int v = e * 256 + threadIdx.x;
            const int row = v >> 6, col = v & 63;
            const int64_t i = i0 + row, j = j0 + col;
            if (i < rows && j < cols) {
                const int64_t idx = i * cols + j;
                float g;
                if (!PARTS) {
                    g = load_elem(gradp, idx, gbf);
                } else {
                    g = load_elem(parts[0], idx, gbf);
                    for (int r = 1; r < nparts; ++r) g += load_elem(parts[r], idx, gbf);
                }
                const float b = beta * bufp[idx] + omb * g;
                const float m = sc.nesterov ? (omb * g + beta * b) : b;
                bufp[idx] = b;
                sumsq += m * m;
                if (!tr) {
                    if (bf16_mode) store1_master(xb, xl, i * ldx + j, m);
                    else xf[i * ldx + j] = m;
                } else {
                    tileM[row][col] = m;
                }
            }
        }
    }
    if (tr) {
        __syncthreads();
        // X = M^T: X[j][i] = M[i][j]; a thread writes 4 consecutive i of one X row
        if (full && mom_vec) {
            #pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int v = e * 256 + threadIdx.x;
                const int orow = v >> 4, oc = (v & 15) * 4;     // X row = M col, X cols oc..oc+3 = M rows
                const float4 m = make_float4(tileM[oc][orow], tileM[oc + 1][orow], tileM[oc + 2][orow],
                                             tileM[oc + 3][orow]);
                const int64_t xi = (j0 + orow) * ldx + i0 + oc;
                if (bf16_mode) store4_master(xb, xl, xi, m);
                else *reinterpret_cast<float4*>(xf + xi) = m;
            }
        } else {
            for (int e = 0; e < 16; ++e) {
                const int v = e * 256 + threadIdx.x;
                const int orow = v >> 6, ocol = v & 63;   // X row = M col, X col = M row
                const int64_t xr = j0 + orow, xc = i0 + ocol;
                if (xr < cols && xc < rows) {
                    const float m = tileM[ocol][orow];
                    if (bf16_mode) store1_master(xb, xl, xr * ldx + xc, m);
                    else xf[xr * ldx + xc] = m;
                }
            }
        }
    }
    }
    const float tot = block_sum(sumsq, red);
    if (threadIdx.x == 0) partials[grp] = tot;
}

// K1 on flat matrices: one group (kFlatGroup contiguous elements of M and X) per
// block of 256 threads, the group's sum of M^2 to partials[grp].  Three blocks
// per SM leave each thread room for four runs of loads in flight.
template <bool PARTS>
__global__ void __launch_bounds__(256, 3)
momentum_flat_kernel(const MatDev* __restrict__ mats, int nmats, StepScalars sc, float* __restrict__ partials,
                     int32_t* status) {
    __shared__ float red[8];
    const int grp = blockIdx.x;
    const int mi = find_matrix(mats, nmats, grp);
    const MatDev& md = mats[mi];
    if (grp < md.mom_grp0 || !md.mom_flat) {  // cannot happen with a host-built table
        record_status(status, -7);
        return;
    }
    const int64_t e0 = (int64_t)(grp - md.mom_grp0) * kFlatGroup;
    const int64_t n = md.rows * md.cols;
    float sumsq;
    if (PARTS)
        sumsq = momentum_flat<2, true, false>(md, sc, md.buf, md.grad, md.gparts, md.nparts, e0, n);
    else if (md.grad_bf16)
        sumsq = momentum_flat<4, false, true>(md, sc, md.buf, md.grad, md.gparts, md.nparts, e0, n);
    else
        sumsq = momentum_flat<2, false, false>(md, sc, md.buf, md.grad, md.gparts, md.nparts, e0, n);
    const float tot = block_sum(sumsq, red);
    if (threadIdx.x == 0) partials[grp] = tot;
}

// ---------------------------------------------------------------------------
// Flat groups through 1D bulk copies (TMA): one thread streams a group's inputs
// into a 3-stage shared-memory ring in runs of kBulkSub elements, the block
// computes from shared memory and stores straight to global memory.  The
// loads in flight cost no registers, so six blocks per SM keep up to 216 KB of
// them in flight.  Every wait is bounded; on a timeout the block records
// MFSDP_ERR_TIMEOUT, waits (bounded) for its own copies still in flight and
// returns.
// ---------------------------------------------------------------------------
constexpr int kBulkSub = 2048;                  // elements per stage (one run of 8 per thread)
constexpr int kBulkStages = 3;
constexpr int kBulkSubs = kFlatGroup / kBulkSub;
constexpr unsigned long long kBulkWaitNs = 1000000000ull;   // 1 s per wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void bulk_bar_init(uint32_t bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void bulk_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// global -> shared, `bytes` a multiple of 16, both addresses 16-byte aligned
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ bool bulk_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(100000u)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long bulk_clock() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ bool bulk_wait(uint32_t bar, uint32_t parity, unsigned long long limit_ns) {
    const unsigned long long t0 = bulk_clock();
    while (!bulk_try_wait(bar, parity))
        if (bulk_clock() - t0 > limit_ns) return false;
    return true;
}

// The ring of one block: stage s of run k holds run k's slice of each input.
// Thread 0 issues run k into stage k % kBulkStages once the block is done with
// run k - kBulkStages; every thread waits for run k before using it.
struct BulkRing {
    uint64_t bar[kBulkStages];
    int abort;
};

// Waits for run k (thread 0 polls, the block follows).  False on a timeout: the
// block then drains (thread 0 waits, bounded, for the copies it issued) and stops.
__device__ __forceinline__ bool bulk_ring_wait(BulkRing& ring, int k, int issued, int32_t* status) {
    if (threadIdx.x == 0) {
        const bool ok = bulk_wait(smem_u32(&ring.bar[k % kBulkStages]), (k / kBulkStages) & 1, kBulkWaitNs);
        if (!ok) {
            ring.abort = 1;
            record_status(status, -6 /* MFSDP_ERR_TIMEOUT */);
            for (int j = k; j < issued; ++j)   // the copies still in flight
                (void)bulk_wait(smem_u32(&ring.bar[j % kBulkStages]), (j / kBulkStages) & 1, 10000000ull);
        }
    }
    __syncthreads();
    return ring.abort == 0;
}

// Momentum on one flat group with bf16 gradients (not the owner-segment sum).
__global__ void __launch_bounds__(256)
momentum_bulk_kernel(const MatDev* __restrict__ mats, int nmats, StepScalars sc, float* __restrict__ partials,
                     int32_t* status) {
    __shared__ __align__(128) float sbuf[kBulkStages][kBulkSub];
    __shared__ __align__(128) __nv_bfloat16 sgrad[kBulkStages][kBulkSub];
    __shared__ BulkRing ring;
    __shared__ float red[8];
    const int grp = blockIdx.x;
    const int mi = find_matrix(mats, nmats, grp);
    const MatDev& md = mats[mi];
    if (grp < md.mom_grp0 || !md.mom_flat || !md.grad_bf16) {   // cannot happen with a host-built table
        record_status(status, -7);
        return;
    }
    const int64_t n = md.rows * md.cols;
    const int64_t e0 = (int64_t)(grp - md.mom_grp0) * kFlatGroup;
    const int64_t left = n - e0;                      // a multiple of 8, > 0
    const int runs = static_cast<int>(min((int64_t)kBulkSubs, (left + kBulkSub - 1) / kBulkSub));
    float* __restrict__ bufp = md.buf;
    const __nv_bfloat16* gradp = static_cast<const __nv_bfloat16*>(md.grad);
    auto issue = [&](int k) {                         // thread 0
        const int64_t i0 = e0 + (int64_t)k * kBulkSub;
        const uint32_t cnt = static_cast<uint32_t>(min((int64_t)kBulkSub, n - i0));
        const uint32_t bar = smem_u32(&ring.bar[k % kBulkStages]);
        bulk_expect(bar, cnt * 6);
        bulk_load(smem_u32(sbuf[k % kBulkStages]), bufp + i0, cnt * 4, bar);
        bulk_load(smem_u32(sgrad[k % kBulkStages]), gradp + i0, cnt * 2, bar);
    };
    int issued = 0;
    if (threadIdx.x == 0) {
        ring.abort = 0;
        for (int s = 0; s < kBulkStages; ++s) bulk_bar_init(smem_u32(&ring.bar[s]));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (; issued < min(kBulkStages, runs); ++issued) issue(issued);
    }
    __syncthreads();
    const float beta = sc.beta, omb = 1.0f - sc.beta;
    float sumsq = 0.f;
    for (int k = 0; k < runs; ++k) {
        if (!bulk_ring_wait(ring, k, threadIdx.x == 0 ? issued : 0, status)) return;
        const int st = k % kBulkStages;
        const int64_t base = e0 + (int64_t)k * kBulkSub;
        // two runs of 4 per thread, kBulkSub / 2 apart: conflict-free 16-byte shared reads
        #pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int e = half * (kBulkSub / 2) + 4 * threadIdx.x;   // element within the stage
            const int64_t i = base + e;
            if (i >= n) continue;
            const float4 b = *reinterpret_cast<const float4*>(&sbuf[st][e]);
            const uint2 gq = *reinterpret_cast<const uint2*>(&sgrad[st][e]);
            const float g[4] = {__uint_as_float(gq.x << 16), __uint_as_float(gq.x & 0xFFFF0000u),
                                __uint_as_float(gq.y << 16), __uint_as_float(gq.y & 0xFFFF0000u)};
            const float bin[4] = {b.x, b.y, b.z, b.w};
            float bo[4], m[4];
            #pragma unroll
            for (int j = 0; j < 4; ++j) {
                bo[j] = beta * bin[j] + omb * g[j];
                m[j] = sc.nesterov ? omb * g[j] + beta * bo[j] : bo[j];
                sumsq += m[j] * m[j];
            }
            __stcs(reinterpret_cast<float4*>(bufp + i), make_float4(bo[0], bo[1], bo[2], bo[3]));
            const float4 mv = make_float4(m[0], m[1], m[2], m[3]);
            if (sc.bf16_mode) store4_master(md.xb[0], md.xlo[0], i, mv);
            else *reinterpret_cast<float4*>(md.xf[0] + i) = mv;
        }
        __syncthreads();                              // every thread is done with stage st
        if (threadIdx.x == 0 && issued < runs) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(issued++);
        }
    }
    const float tot = block_sum(sumsq, red);
    if (threadIdx.x == 0) partials[grp] = tot;
}

// The parameter write on one flat group, bf16 mode with a bf16 parameter.
__global__ void __launch_bounds__(256)
param_write_bulk_kernel(const MatDev* __restrict__ mats, int nmats, StepScalars sc, const float* __restrict__ s,
                        int xsel, int use_s, int32_t* status) {
    __shared__ __align__(128) __nv_bfloat16 sxh[kBulkStages][kBulkSub];
    __shared__ __align__(128) __nv_bfloat16 sxl[kBulkStages][kBulkSub];
    __shared__ __align__(128) __nv_bfloat16 sw[kBulkStages][kBulkSub];
    __shared__ BulkRing ring;
    const int grp = blockIdx.x;
    const int mi = find_matrix(mats, nmats, grp);
    const MatDev& md = mats[mi];
    if (grp < md.mom_grp0 || !md.mom_flat || !md.param_bf16 || !sc.bf16_mode) {
        record_status(status, -7);
        return;
    }
    const int64_t n = md.rows * md.cols;
    const int64_t e0 = (int64_t)(grp - md.mom_grp0) * kFlatGroup;
    const int64_t left = n - e0;
    const int runs = static_cast<int>(min((int64_t)kBulkSubs, (left + kBulkSub - 1) / kBulkSub));
    const __nv_bfloat16* xh = md.xb[xsel];
    const __nv_bfloat16* xl = md.xlo[xsel];
    __nv_bfloat16* wp = static_cast<__nv_bfloat16*>(md.param);
    auto issue = [&](int k) {
        const int64_t i0 = e0 + (int64_t)k * kBulkSub;
        const uint32_t cnt = static_cast<uint32_t>(min((int64_t)kBulkSub, n - i0));
        const uint32_t bar = smem_u32(&ring.bar[k % kBulkStages]);
        bulk_expect(bar, cnt * 6);
        bulk_load(smem_u32(sxh[k % kBulkStages]), xh + i0, cnt * 2, bar);
        bulk_load(smem_u32(sxl[k % kBulkStages]), xl + i0, cnt * 2, bar);
        bulk_load(smem_u32(sw[k % kBulkStages]), wp + i0, cnt * 2, bar);
    };
    int issued = 0;
    if (threadIdx.x == 0) {
        ring.abort = 0;
        for (int st = 0; st < kBulkStages; ++st) bulk_bar_init(smem_u32(&ring.bar[st]));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (; issued < min(kBulkStages, runs); ++issued) issue(issued);
    }
    __syncthreads();
    const float f = md.shape_scale * (use_s ? s[mi] : 1.0f);
    const float lr = sc.lr, decay = sc.decay;
    float* __restrict__ uo = md.update_out;
    void* const* copies = md.pcopies;
    const int ncopies = md.ncopies;
    for (int k = 0; k < runs; ++k) {
        if (!bulk_ring_wait(ring, k, threadIdx.x == 0 ? issued : 0, status)) return;
        const int st = k % kBulkStages;
        const int64_t i = e0 + (int64_t)k * kBulkSub + 8 * threadIdx.x;
        if (i < n) {
            const uint4 h = reinterpret_cast<const uint4*>(sxh[st])[threadIdx.x];
            const uint4 l = reinterpret_cast<const uint4*>(sxl[st])[threadIdx.x];
            const uint4 wq = reinterpret_cast<const uint4*>(sw[st])[threadIdx.x];
            const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, lw[4] = {l.x, l.y, l.z, l.w};
            const uint32_t ww[4] = {wq.x, wq.y, wq.z, wq.w};
            float o[8];
            uint32_t nw[4];
            #pragma unroll
            for (int j = 0; j < 4; ++j) {
                o[2 * j] = f * master_value(static_cast<uint16_t>(hw[j] & 0xFFFFu), static_cast<uint16_t>(lw[j] & 0xFFFFu));
                o[2 * j + 1] = f * master_value(static_cast<uint16_t>(hw[j] >> 16), static_cast<uint16_t>(lw[j] >> 16));
                const float w0 = __uint_as_float(ww[j] << 16), w1 = __uint_as_float(ww[j] & 0xFFFF0000u);
                const __nv_bfloat162 p2 = __floats2bfloat162_rn(fmaf(-lr, o[2 * j], w0 * decay),
                                                                fmaf(-lr, o[2 * j + 1], w1 * decay));
                nw[j] = *reinterpret_cast<const uint32_t*>(&p2);
            }
            const uint4 out = make_uint4(nw[0], nw[1], nw[2], nw[3]);
            *reinterpret_cast<uint4*>(wp + i) = out;
            for (int d = 0; d < ncopies; ++d) *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(copies[d]) + i) = out;
            if (uo) {
                *reinterpret_cast<float4*>(uo + i) = make_float4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<float4*>(uo + i + 4) = make_float4(o[4], o[5], o[6], o[7]);
            }
        }
        __syncthreads();
        if (threadIdx.x == 0 && issued < runs) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(issued++);
        }
    }
}

// K2: s = 1 / (||M||_F + eps) per matrix; fixed-order fp64 sum of the group partials.
__global__ void __launch_bounds__(256)
norm_kernel(const MatDev* __restrict__ mats, int nmats, const float* __restrict__ partials,
            float* __restrict__ s_out, float eps) {
    __shared__ double red[8];
    const int mi = blockIdx.x;
    if (mi >= nmats) return;
    const MatDev& md = mats[mi];
    const int64_t groups = md.mom_groups_n;
    double acc = 0.0;
    for (int64_t g = threadIdx.x; g < groups; g += blockDim.x) acc += (double)partials[md.mom_grp0 + g];
    const double tot = block_sum(acc, red);
    if (threadIdx.x == 0) s_out[mi] = (float)(1.0 / (sqrt(tot) + (double)eps));
}

// Parameter write, one 64 x 64 tile of W per block (the momentum tiling):
//   O = f * X (transposed back when rows > cols),  W <- W (1 - lr wd) - lr O
// with f = shape scale, times s when no Newton-Schulz iteration ran (X is then
// the unnormalised M).  X comes from master copy `xsel` (hi part and remainder
// in bf16 mode, fp32 in fp32 mode).  A
// transposed X tile goes through shared memory so both X and W are read and
// written along their rows; full tiles move 4 elements per access.
__global__ void __launch_bounds__(256, 4)
param_write_kernel(const MatDev* __restrict__ mats, int nmats, int grp_base, StepScalars sc,
                   const float* __restrict__ s, int xsel, int use_s, int32_t* status) {
    // transposed tiles alternate between two staging tiles: one block barrier per tile
    __shared__ float tileX2[2][kMomTile][kMomTile + 1];
    const int grp = grp_base + blockIdx.x;
    const int mi = find_matrix(mats, nmats, grp);
    const MatDev& md = mats[mi];
    const int64_t rows = md.rows, cols = md.cols;
    const int tiles_n = md.mom_tiles_n, grp0 = md.mom_grp0;
    const int64_t ntiles = ((rows + kMomTile - 1) / kMomTile) * tiles_n;
    if (grp < grp0) {
        record_status(status, -7);
        return;
    }
    const bool tr = md.tr != 0;
    const float f = md.shape_scale * (use_s ? s[mi] : 1.0f);
    const float lr = sc.lr, decay = sc.decay;
    const bool bfm = sc.bf16_mode != 0;         // X as hi + remainder (bf16 mode) or fp32
    const float* __restrict__ xf = md.xf[xsel];
    const __nv_bfloat16* __restrict__ xb = md.xb[xsel];
    const __nv_bfloat16* __restrict__ xl = md.xlo[xsel];
    const int64_t ldx = md.ldx;
    const bool wbf = md.param_bf16 != 0;
    float* wf = static_cast<float*>(md.param);
    __nv_bfloat16* wb = static_cast<__nv_bfloat16*>(md.param);
    float* uo = md.update_out;
    void* const* copies = md.pcopies;        // owner-segment destinations of the new parameter
    const int ncopies = md.ncopies;
    bool aligned_w = (cols % 4 == 0) && (reinterpret_cast<uintptr_t>(md.param) % (wbf ? 8 : 16) == 0) &&
                     (uo == nullptr || reinterpret_cast<uintptr_t>(uo) % 16 == 0);
    for (int d = 0; d < ncopies; ++d)
        aligned_w = aligned_w && (reinterpret_cast<uintptr_t>(copies[d]) % (wbf ? 8 : 16) == 0);
    // bf16 mode with a bf16 parameter: 8 elements per access (one 16-byte load
    // each of X's hi part, X's lo part and W)
    bool wide = bfm && wbf && (cols % 8 == 0) && (reinterpret_cast<uintptr_t>(md.param) % 16 == 0) &&
                (uo == nullptr || reinterpret_cast<uintptr_t>(uo) % 16 == 0);
    for (int d = 0; d < ncopies; ++d) wide = wide && (reinterpret_cast<uintptr_t>(copies[d]) % 16 == 0);

    for (int k = 0; k < kMomGroup; ++k) {
    const int local = (grp - grp0) * kMomGroup + k;
    if (local >= ntiles) break;      // block-uniform
    const int sb = k & 1;            // staging tile of this tile
    const int ti = local / tiles_n, tj = local % tiles_n;
    const int64_t i0 = (int64_t)ti * kMomTile, j0 = (int64_t)tj * kMomTile;   // W tile origin
    const bool full = (i0 + kMomTile <= rows) && (j0 + kMomTile <= cols);
    if (full && wide) {
        // thread: rows v >> 3 of the tile, 8 columns from (v & 7) * 8, for v = tid, tid + 256
        float xv[2][8];
        uint4 wv[2];
        if (tr) {
            #pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int v = e * 256 + threadIdx.x;
                const int xr = v >> 3, xc = (v & 7) * 8;       // X tile row (a W column), 8 X columns (W rows)
                const int64_t xi = (j0 + xr) * ldx + i0 + xc;
                const uint4 h = __ldg(reinterpret_cast<const uint4*>(xb + xi));
                const uint4 l = __ldg(reinterpret_cast<const uint4*>(xl + xi));
                const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, lw[4] = {l.x, l.y, l.z, l.w};
                #pragma unroll
                for (int u = 0; u < 4; ++u) {
                    tileX2[sb][xr][xc + 2 * u] = master_value(static_cast<uint16_t>(hw[u] & 0xFFFFu),
                                                         static_cast<uint16_t>(lw[u] & 0xFFFFu));
                    tileX2[sb][xr][xc + 2 * u + 1] = master_value(static_cast<uint16_t>(hw[u] >> 16),
                                                             static_cast<uint16_t>(lw[u] >> 16));
                }
            }
        }
        #pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int v = e * 256 + threadIdx.x;
            const int row = v >> 3, col = (v & 7) * 8;
            wv[e] = *reinterpret_cast<const uint4*>(wb + (i0 + row) * cols + j0 + col);   // written below: no .nc
            if (!tr) {
                const int64_t xi = (i0 + row) * ldx + j0 + col;
                const uint4 h = __ldg(reinterpret_cast<const uint4*>(xb + xi));
                const uint4 l = __ldg(reinterpret_cast<const uint4*>(xl + xi));
                const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, lw[4] = {l.x, l.y, l.z, l.w};
                #pragma unroll
                for (int u = 0; u < 4; ++u) {
                    xv[e][2 * u] = master_value(static_cast<uint16_t>(hw[u] & 0xFFFFu), static_cast<uint16_t>(lw[u] & 0xFFFFu));
                    xv[e][2 * u + 1] = master_value(static_cast<uint16_t>(hw[u] >> 16), static_cast<uint16_t>(lw[u] >> 16));
                }
            }
        }
        if (tr) {
            __syncthreads();
            #pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int v = e * 256 + threadIdx.x;
                const int row = v >> 3, col = (v & 7) * 8;
                #pragma unroll
                for (int u = 0; u < 8; ++u) xv[e][u] = tileX2[sb][col + u][row];
            }
        }
        #pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int v = e * 256 + threadIdx.x;
            const int row = v >> 3, col = (v & 7) * 8;
            const int64_t widx = (i0 + row) * cols + j0 + col;
            const uint32_t ww[4] = {wv[e].x, wv[e].y, wv[e].z, wv[e].w};
            uint32_t nw[4];
            float o[8];
            #pragma unroll
            for (int u = 0; u < 4; ++u) {
                o[2 * u] = f * xv[e][2 * u];
                o[2 * u + 1] = f * xv[e][2 * u + 1];
                const float w0 = __uint_as_float(ww[u] << 16), w1 = __uint_as_float(ww[u] & 0xFFFF0000u);
                const __nv_bfloat162 n = __floats2bfloat162_rn(fmaf(-lr, o[2 * u], w0 * decay),
                                                               fmaf(-lr, o[2 * u + 1], w1 * decay));
                nw[u] = *reinterpret_cast<const uint32_t*>(&n);
            }
            const uint4 out = make_uint4(nw[0], nw[1], nw[2], nw[3]);
            *reinterpret_cast<uint4*>(wb + widx) = out;
            if (uo) {
                *reinterpret_cast<float4*>(uo + widx) = make_float4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<float4*>(uo + widx + 4) = make_float4(o[4], o[5], o[6], o[7]);
            }
            for (int d = 0; d < ncopies; ++d) *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(copies[d]) + widx) = out;
        }
        continue;
    }
    if (tr) {
        // X tile rows = W columns j0.., X tile columns = W rows i0..
        if (full && (ldx % 4 == 0)) {
            #pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int v = e * 256 + threadIdx.x;
                const int xr = v >> 4, xc = (v & 15) * 4;
                const int64_t xi = (j0 + xr) * ldx + i0 + xc;
                const float4 x = bfm ? load4_master(xb, xl, xi) : *reinterpret_cast<const float4*>(xf + xi);
                tileX2[sb][xr][xc] = x.x; tileX2[sb][xr][xc + 1] = x.y; tileX2[sb][xr][xc + 2] = x.z; tileX2[sb][xr][xc + 3] = x.w;
            }
        } else {
            for (int e = 0; e < 16; ++e) {
                const int v = e * 256 + threadIdx.x;
                const int xr = v >> 6, xc = v & 63;
                if (j0 + xr < cols && i0 + xc < rows) {
                    const int64_t xi = (j0 + xr) * ldx + i0 + xc;
                    tileX2[sb][xr][xc] = bfm ? load1_master(xb, xl, xi) : xf[xi];
                }
            }
        }
        __syncthreads();
    }
    if (full && aligned_w) {
        // every load of this thread is issued before any store
        float4 xv[4], wv[4];
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int v = e * 256 + threadIdx.x;
            const int row = v >> 4, col = (v & 15) * 4;
            if (tr) xv[e] = make_float4(tileX2[sb][col][row], tileX2[sb][col + 1][row], tileX2[sb][col + 2][row], tileX2[sb][col + 3][row]);
            else if (bfm) xv[e] = load4_master(xb, xl, (i0 + row) * ldx + j0 + col);
            else xv[e] = *reinterpret_cast<const float4*>(xf + (i0 + row) * ldx + j0 + col);
            wv[e] = load4(md.param, (i0 + row) * cols + j0 + col, wbf);
        }
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int v = e * 256 + threadIdx.x;
            const int row = v >> 4, col = (v & 15) * 4;
            const int64_t widx = (i0 + row) * cols + j0 + col;
            const float4 o = make_float4(f * xv[e].x, f * xv[e].y, f * xv[e].z, f * xv[e].w);
            float4 w = wv[e];
            w.x = fmaf(-lr, o.x, w.x * decay); w.y = fmaf(-lr, o.y, w.y * decay);
            w.z = fmaf(-lr, o.z, w.z * decay); w.w = fmaf(-lr, o.w, w.w * decay);
            if (wbf) store4_bf16(wb, widx, w);
            else *reinterpret_cast<float4*>(wf + widx) = w;
            if (uo) *reinterpret_cast<float4*>(uo + widx) = o;
            for (int d = 0; d < ncopies; ++d) {
                if (wbf) store4_bf16(static_cast<__nv_bfloat16*>(copies[d]), widx, w);
                else *reinterpret_cast<float4*>(static_cast<float*>(copies[d]) + widx) = w;
            }
        }
    } else {
    for (int e = 0; e < 16; ++e) {
        const int v = e * 256 + threadIdx.x;
        const int row = v >> 6, col = v & 63;
        const int64_t i = i0 + row, j = j0 + col;
        if (i >= rows || j >= cols) continue;
        const float x = tr ? tileX2[sb][col][row] : (bfm ? load1_master(xb, xl, i * ldx + j) : xf[i * ldx + j]);
        const float o = f * x;
        const int64_t idx = i * cols + j;
        if (uo) uo[idx] = o;
        if (wbf) {
            const __nv_bfloat16 nw = __float2bfloat16_rn(fmaf(-lr, o, __bfloat162float(wb[idx]) * decay));
            wb[idx] = nw;
            for (int d = 0; d < ncopies; ++d) static_cast<__nv_bfloat16*>(copies[d])[idx] = nw;
        } else {
            const float nw = fmaf(-lr, o, wf[idx] * decay);
            wf[idx] = nw;
            for (int d = 0; d < ncopies; ++d) static_cast<float*>(copies[d])[idx] = nw;
        }
    }
    }
    }
}

// The parameter write on flat matrices: one group (kFlatGroup contiguous elements
// of W and X, the momentum kernel's groups) per block, runs of 8 elements, U runs
// of raw loads in flight (bf16 values stay packed until used).
//   BFM: X is the bf16 hi + lo master (else fp32);  WBF: W is bf16 (else fp32).
template <int U, bool BFM, bool WBF>
__device__ __forceinline__ void param_write_flat(const MatDev& md, const StepScalars& sc, float f,
                                                 const float* __restrict__ xf, const __nv_bfloat16* __restrict__ xb,
                                                 const __nv_bfloat16* __restrict__ xl, int64_t e0, int64_t n) {
    const float lr = sc.lr, decay = sc.decay;
    float* __restrict__ uo = md.update_out;
    void* const* copies = md.pcopies;
    const int ncopies = md.ncopies;
    #pragma unroll 1
    for (int c0 = 0; c0 < kFlatGroup / 8; c0 += U * 256) {
        uint4 xq[U][2], wq[U][2];
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = e0 + 8 * (int64_t)(c0 + u * 256 + threadIdx.x);
            if (i >= n) continue;
            if (BFM) {
                xq[u][0] = __ldcs(reinterpret_cast<const uint4*>(xb + i));
                xq[u][1] = __ldcs(reinterpret_cast<const uint4*>(xl + i));
            } else {
                xq[u][0] = __ldcs(reinterpret_cast<const uint4*>(xf + i));
                xq[u][1] = __ldcs(reinterpret_cast<const uint4*>(xf + i) + 1);
            }
            // W is written below: no streaming or read-only hint on its load
            if (WBF) {
                wq[u][0] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(md.param) + i);
            } else {
                wq[u][0] = *reinterpret_cast<const uint4*>(static_cast<const float*>(md.param) + i);
                wq[u][1] = *(reinterpret_cast<const uint4*>(static_cast<const float*>(md.param) + i) + 1);
            }
        }
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = e0 + 8 * (int64_t)(c0 + u * 256 + threadIdx.x);
            if (i >= n) continue;
            float x[8], w[8];
            const uint32_t a[4] = {xq[u][0].x, xq[u][0].y, xq[u][0].z, xq[u][0].w};
            const uint32_t b[4] = {xq[u][1].x, xq[u][1].y, xq[u][1].z, xq[u][1].w};
            #pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (BFM) {
                    x[2 * k] = master_value(static_cast<uint16_t>(a[k] & 0xFFFFu), static_cast<uint16_t>(b[k] & 0xFFFFu));
                    x[2 * k + 1] = master_value(static_cast<uint16_t>(a[k] >> 16), static_cast<uint16_t>(b[k] >> 16));
                } else {
                    x[k] = __uint_as_float(a[k]);
                    x[k + 4] = __uint_as_float(b[k]);
                }
            }
            const uint32_t wa[4] = {wq[u][0].x, wq[u][0].y, wq[u][0].z, wq[u][0].w};
            const uint32_t wb2[4] = {wq[u][1].x, wq[u][1].y, wq[u][1].z, wq[u][1].w};
            #pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (WBF) {
                    w[2 * k] = __uint_as_float(wa[k] << 16);
                    w[2 * k + 1] = __uint_as_float(wa[k] & 0xFFFF0000u);
                } else {
                    w[k] = __uint_as_float(wa[k]);
                    w[k + 4] = __uint_as_float(wb2[k]);
                }
            }
            float o[8];
            #pragma unroll
            for (int k = 0; k < 8; ++k) {
                o[k] = f * x[k];
                w[k] = fmaf(-lr, o[k], w[k] * decay);
            }
            if (WBF) {
                uint32_t nw[4];
                #pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const __nv_bfloat162 p2 = __floats2bfloat162_rn(w[2 * k], w[2 * k + 1]);
                    nw[k] = *reinterpret_cast<const uint32_t*>(&p2);
                }
                const uint4 out = make_uint4(nw[0], nw[1], nw[2], nw[3]);
                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(md.param) + i) = out;
                for (int d = 0; d < ncopies; ++d) *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(copies[d]) + i) = out;
            } else {
                const float4 lo = make_float4(w[0], w[1], w[2], w[3]), hi = make_float4(w[4], w[5], w[6], w[7]);
                *reinterpret_cast<float4*>(static_cast<float*>(md.param) + i) = lo;
                *(reinterpret_cast<float4*>(static_cast<float*>(md.param) + i) + 1) = hi;
                for (int d = 0; d < ncopies; ++d) {
                    *reinterpret_cast<float4*>(static_cast<float*>(copies[d]) + i) = lo;
                    *(reinterpret_cast<float4*>(static_cast<float*>(copies[d]) + i) + 1) = hi;
                }
            }
            if (uo) {
                *reinterpret_cast<float4*>(uo + i) = make_float4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<float4*>(uo + i + 4) = make_float4(o[4], o[5], o[6], o[7]);
            }
        }
    }
}

__global__ void __launch_bounds__(256, 3)
param_write_flat_kernel(const MatDev* __restrict__ mats, int nmats, StepScalars sc, const float* __restrict__ s,
                        int xsel, int use_s, int32_t* status) {
    const int grp = blockIdx.x;
    const int mi = find_matrix(mats, nmats, grp);
    const MatDev& md = mats[mi];
    if (grp < md.mom_grp0 || !md.mom_flat) {  // cannot happen with a host-built table
        record_status(status, -7);
        return;
    }
    const int64_t e0 = (int64_t)(grp - md.mom_grp0) * kFlatGroup;
    const int64_t n = md.rows * md.cols;
    const float f = md.shape_scale * (use_s ? s[mi] : 1.0f);
    const bool wbf = md.param_bf16 != 0;
    if (sc.bf16_mode) {
        if (wbf) param_write_flat<4, true, true>(md, sc, f, md.xf[xsel], md.xb[xsel], md.xlo[xsel], e0, n);
        else param_write_flat<2, true, false>(md, sc, f, md.xf[xsel], md.xb[xsel], md.xlo[xsel], e0, n);
    } else {
        if (wbf) param_write_flat<2, false, true>(md, sc, f, md.xf[xsel], md.xb[xsel], md.xlo[xsel], e0, n);
        else param_write_flat<2, false, false>(md, sc, f, md.xf[xsel], md.xb[xsel], md.xlo[xsel], e0, n);
    }
}

// ---------------------------------------------------------------------------
// K6: AdamW over the packed fp32 tail.  28 algorithmic bytes per element.
// ---------------------------------------------------------------------------
struct AdamScalars {
    float lr, beta1, beta2, eps, decay, bc1, bc2;
};

__device__ __forceinline__ void adam_elem(float& p, float g, float& m, float& v, const AdamScalars& a) {
    m = a.beta1 * m + (1.0f - a.beta1) * g;
    v = a.beta2 * v + (1.0f - a.beta2) * (g * g);
    const float mhat = m / a.bc1;
    const float vhat = v / a.bc2;
    p = p * a.decay - a.lr * mhat / (sqrtf(vhat) + a.eps);
}

// Four 16-byte groups of each of p, g, m, v in flight per thread (16 loads)
// before any arithmetic; streaming hints keep the one-pass tail from
// displacing L2 contents.
__global__ void __launch_bounds__(256)
adamw_vec_kernel(float4* __restrict__ p, const float4* __restrict__ g, float4* __restrict__ m,
                 float4* __restrict__ v, int64_t n4, AdamScalars a) {
    constexpr int U = 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < n4; i0 += U * stride) {
        float4 P[U], G[U], M[U], V[U];
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < n4) {
                P[u] = __ldcs(p + i); G[u] = __ldcs(g + i); M[u] = __ldcs(m + i); V[u] = __ldcs(v + i);
            }
        }
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < n4) {
                adam_elem(P[u].x, G[u].x, M[u].x, V[u].x, a); adam_elem(P[u].y, G[u].y, M[u].y, V[u].y, a);
                adam_elem(P[u].z, G[u].z, M[u].z, V[u].z, a); adam_elem(P[u].w, G[u].w, M[u].w, V[u].w, a);
                __stcs(p + i, P[u]); __stcs(m + i, M[u]); __stcs(v + i, V[u]);
            }
        }
    }
}

__global__ void __launch_bounds__(256)
adamw_scalar_kernel(float* __restrict__ p, const float* __restrict__ g, float* __restrict__ m,
                    float* __restrict__ v, int64_t n, AdamScalars a) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        float P = p[i], M = m[i], V = v[i];
        adam_elem(P, g[i], M, V, a);
        p[i] = P; m[i] = M; v[i] = V;
    }
}

int sm_count() {
    // initialised once, thread-safely, on the first call
    static const int count = [] {
        int dev = 0, c = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) {
            cudaGetLastError();
            c = 148;
        }
        return c;
    }();
    return count;
}

}  // namespace

cudaError_t launch_momentum(const MatDev* d_mats, int32_t nmats, int32_t flat_groups, int32_t total_groups,
                            const StepScalars& sc, float* partials, bool parts, bool flat_bulk, cudaStream_t st) {
    if (flat_groups > 0) {
        if (parts)
            momentum_flat_kernel<true><<<flat_groups, 256, 0, st>>>(d_mats, nmats, sc, partials, device_status_ptr());
        else if (flat_bulk)
            momentum_bulk_kernel<<<flat_groups, 256, 0, st>>>(d_mats, nmats, sc, partials, device_status_ptr());
        else
            momentum_flat_kernel<false><<<flat_groups, 256, 0, st>>>(d_mats, nmats, sc, partials, device_status_ptr());
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int32_t tiled = total_groups - flat_groups;
    if (tiled > 0) {
        if (parts)
            momentum_kernel<true><<<tiled, 256, 0, st>>>(d_mats, nmats, flat_groups, sc, partials, device_status_ptr());
        else
            momentum_kernel<false><<<tiled, 256, 0, st>>>(d_mats, nmats, flat_groups, sc, partials, device_status_ptr());
    }
    return cudaGetLastError();
}

cudaError_t launch_norm(const MatDev* d_mats, int32_t nmats, const float* partials,
                        float* s_out, float eps, cudaStream_t st) {
    if (nmats <= 0) return cudaSuccess;
    norm_kernel<<<nmats, 256, 0, st>>>(d_mats, nmats, partials, s_out, eps);
    return cudaGetLastError();
}

cudaError_t launch_param_write(const MatDev* d_mats, int32_t nmats, int32_t flat_groups, int32_t total_groups,
                               const StepScalars& sc, const float* s, int32_t xsel, int32_t use_s, bool flat_bulk,
                               cudaStream_t st) {
    if (flat_groups > 0) {
        if (flat_bulk)
            param_write_bulk_kernel<<<flat_groups, 256, 0, st>>>(d_mats, nmats, sc, s, xsel, use_s, device_status_ptr());
        else
            param_write_flat_kernel<<<flat_groups, 256, 0, st>>>(d_mats, nmats, sc, s, xsel, use_s, device_status_ptr());
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int32_t tiled = total_groups - flat_groups;
    if (tiled > 0)
        param_write_kernel<<<tiled, 256, 0, st>>>(d_mats, nmats, flat_groups, sc, s, xsel, use_s, device_status_ptr());
    return cudaGetLastError();
}

cudaError_t launch_adamw(float* p, const float* g, float* m, float* v, int64_t n,
                         float lr, float beta1, float beta2, float eps, float decay,
                         float bc1, float bc2, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    AdamScalars a{lr, beta1, beta2, eps, decay, bc1, bc2};
    const bool vec = (n % 4 == 0) &&
                     ((reinterpret_cast<uintptr_t>(p) | reinterpret_cast<uintptr_t>(g) |
                       reinterpret_cast<uintptr_t>(m) | reinterpret_cast<uintptr_t>(v)) % 16 == 0);
    const int64_t work = vec ? n / 4 : n;
    int64_t blocks = (work + 4 * 256 - 1) / (4 * 256);
    // a grid of resident blocks only: the grid-stride loop then has no tail wave
    static const int per_sm = [] {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, adamw_vec_kernel, 256, 0) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 2;
        }
        return n;
    }();
    const int64_t cap = (int64_t)sm_count() * per_sm;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (vec) {
        adamw_vec_kernel<<<(unsigned)blocks, 256, 0, st>>>(
            reinterpret_cast<float4*>(p), reinterpret_cast<const float4*>(g),
            reinterpret_cast<float4*>(m), reinterpret_cast<float4*>(v), work, a);
    } else {
        adamw_scalar_kernel<<<(unsigned)blocks, 256, 0, st>>>(p, g, m, v, n, a);
    }
    return cudaGetLastError();
}

}  // namespace mfsdp
