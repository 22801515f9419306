// Grouped Newton-Schulz GEMM phases on the FFMA pipe (CUDA cores).
//
// This is the engine of fp32 mode only (MFSDP_MODE_FP32: fp32 operands, no
// tf32); bf16 mode always runs on the tcgen05 engine.  One 128 x 128 output
// tile per block of 256 threads, 8 x 8 accumulators per thread, K staged through double-buffered
// shared memory 8 deep.  Phases (one launch each, grouped over all matrices):
//   PH_GRAM   A = s^2 X X^T       upper-triangle tiles, mirrored store
//   PH_POLY   B = b A + c A A     upper-triangle tiles, mirrored store (A symmetric, so A A = A A^T)
//   PH_APPLY  X <- s (a X + B X)
//   PH_FINAL  the same X update into the fp32 master only (the parameter write follows)
// in the diagonal-split form of internal.h: the GEMM operands are the
// zero-diagonal parts E_A, E_B; the diagonals d_A, d_B enter in fp32 epilogues.
// s is the Frobenius scale 1/(||M||+eps) on the first iteration and 1 after:
// the momentum kernel stores M unnormalised and the scale is folded here.
#include "internal.h"

namespace mfsdp {
namespace {

template <typename T>
__device__ __forceinline__ float4 ld4(const T* p);

template <>
__device__ __forceinline__ float4 ld4<float>(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}

__device__ __forceinline__ void mask4(float4& v, int first, int limit) {
    if (first + 0 >= limit) v.x = 0.f;
    if (first + 1 >= limit) v.y = 0.f;
    if (first + 2 >= limit) v.z = 0.f;
    if (first + 3 >= limit) v.w = 0.f;
}

template <typename T>
__device__ __forceinline__ void store_val(T* p, float v);
template <>
__device__ __forceinline__ void store_val<float>(float* p, float v) { *p = v; }

constexpr int BT = kSimtTile;  // 128
constexpr int BK = 8;
constexpr int LDS = BT + 4;

__global__ void __launch_bounds__(256, 2)
simt_phase_kernel(int32_t ph, const MatDev* __restrict__ mats, int32_t nmats,
                  const TileDev* __restrict__ tiles, int32_t iter, StepScalars sc,
                  const float* __restrict__ s, int32_t* status) {
    using T = float;
    __shared__ __align__(16) float As[2][BK][LDS];
    __shared__ __align__(16) float Bs[2][BK][LDS];

    const TileDev t = tiles[blockIdx.x];
    if (t.mat < 0 || t.mat >= nmats) {
        if (threadIdx.x == 0 && status) atomicCAS(status, 0, -7);
        return;
    }
    const MatDev& md = mats[t.mat];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int cur = iter & 1, nxt = cur ^ 1;

    const T* Aop;
    const T* Bop;
    int64_t ldA, ldB;
    int K, Mrows, Ncols;
    const bool gemm = (ph == PH_APPLY || ph == PH_FINAL);
    if (ph == PH_GRAM) {
        Aop = Bop = md.xf[cur];
        ldA = ldB = md.ldx; K = md.c; Mrows = Ncols = md.r;
    } else if (ph == PH_POLY) {
        Aop = Bop = md.af;
        ldA = ldB = md.lda; K = md.r; Mrows = Ncols = md.r;
    } else {
        Aop = reinterpret_cast<const T*>(md.bm);
        ldA = md.lda;
        Bop = md.xf[cur];
        ldB = md.ldx; K = md.r; Mrows = md.r; Ncols = md.c;
    }
    const int i0 = t.tm * BT, j0 = t.tn * BT;

    // loader coordinates
    const int a_row = tid >> 1, a_k = (tid & 1) * 4;       // K-major tile: 128 rows x 8 k
    const int b_k = tid >> 5, b_col = (tid & 31) * 4;       // row-major [k][j] tile: 8 k x 128 j

    auto load_a = [&](int k0, float4& ra) {
        const int row = i0 + a_row, k = k0 + a_k;
        if (row < Mrows && k < K) {
            ra = ld4<T>(Aop + (int64_t)row * ldA + k);
            mask4(ra, k, K);
        } else {
            ra = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto load_b = [&](int k0, float4& rb) {
        if (!gemm) {
            const int row = j0 + a_row, k = k0 + a_k;
            if (row < Ncols && k < K) {
                rb = ld4<T>(Bop + (int64_t)row * ldB + k);
                mask4(rb, k, K);
            } else {
                rb = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        } else {
            const int k = k0 + b_k, col = j0 + b_col;
            if (k < K && col < Ncols) {
                rb = ld4<T>(Bop + (int64_t)k * ldB + col);
                mask4(rb, col, Ncols);
            } else {
                rb = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    };
    auto store_a = [&](int buf, const float4& ra) {
        As[buf][a_k + 0][a_row] = ra.x; As[buf][a_k + 1][a_row] = ra.y;
        As[buf][a_k + 2][a_row] = ra.z; As[buf][a_k + 3][a_row] = ra.w;
    };
    auto store_b = [&](int buf, const float4& rb) {
        if (!gemm) {
            Bs[buf][a_k + 0][a_row] = rb.x; Bs[buf][a_k + 1][a_row] = rb.y;
            Bs[buf][a_k + 2][a_row] = rb.z; Bs[buf][a_k + 3][a_row] = rb.w;
        } else {
            *reinterpret_cast<float4*>(&Bs[buf][b_k][b_col]) = rb;
        }
    };

    float acc[8][8];
    #pragma unroll
    for (int i = 0; i < 8; ++i)
        #pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    const int nk = (K + BK - 1) / BK;
    float4 ra, rb;
    load_a(0, ra); load_b(0, rb);
    store_a(0, ra); store_b(0, rb);
    __syncthreads();
    for (int kt = 0; kt < nk; ++kt) {
        const int b = kt & 1;
        const bool more = kt + 1 < nk;
        if (more) { load_a((kt + 1) * BK, ra); load_b((kt + 1) * BK, rb); }
        #pragma unroll
        for (int k = 0; k < BK; ++k) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[b][k][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[b][k][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[b][k][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[b][k][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            #pragma unroll
            for (int i = 0; i < 8; ++i)
                #pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        if (more) { store_a(b ^ 1, ra); store_b(b ^ 1, rb); }
        __syncthreads();
    }

    // ---- epilogue ----
    const float sg = (iter == 0) ? s[t.mat] : 1.0f;
    #pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int gi = i0 + ((i < 4) ? ty * 4 + i : 64 + ty * 4 + (i - 4));
        if (gi >= Mrows) continue;
        #pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int gj = j0 + ((j < 4) ? tx * 4 + j : 64 + tx * 4 + (j - 4));
            if (gj >= Ncols) continue;
            const float a = acc[i][j];
            if (ph == PH_GRAM) {
                if (gi > gj) continue;
                const float v = (sg * sg) * a;
                if (gi == gj) {
                    md.da[gi] = v;
                    md.af[(int64_t)gi * md.lda + gi] = 0.f;
                } else {
                    md.af[(int64_t)gi * md.lda + gj] = v;
                    md.af[(int64_t)gj * md.lda + gi] = v;
                }
            } else if (ph == PH_POLY) {
                if (gi > gj) continue;
                T* bm = reinterpret_cast<T*>(md.bm);
                const float di = md.da[gi];
                if (gi == gj) {
                    // A_ii = d_i, (A A)_ii = (E E)_ii + d_i^2
                    const float v = sc.b * di + sc.c * fmaf(di, di, a);
                    md.db[gi] = v;
                    store_val<T>(bm + (int64_t)gi * md.lda + gi, 0.f);
                } else {
                    const float e = md.af[(int64_t)gi * md.lda + gj];
                    const float a2 = fmaf(di + md.da[gj], e, a);
                    const float v = sc.b * e + sc.c * a2;
                    store_val<T>(bm + (int64_t)gi * md.lda + gj, v);
                    store_val<T>(bm + (int64_t)gj * md.lda + gi, v);
                }
            } else {
                const int64_t xi = (int64_t)gi * md.ldx + gj;
                const float xin = md.xf[cur][xi];
                const float v = sg * fmaf(sc.a + md.db[gi], xin, a);
                md.xf[nxt][xi] = v;
            }
        }
    }
}

}  // namespace

cudaError_t launch_gemm_simt(Phase ph, const MatDev* d_mats, int32_t nmats, const TileDev* d_tiles, int32_t ntiles,
                             int32_t iter, const StepScalars& sc, const float* s, cudaStream_t st) {
    if (ntiles <= 0) return cudaSuccess;
    if (sc.bf16_mode) return cudaErrorInvalidValue;   // fp32 mode only: its workspace holds fp32 X, A and B
    simt_phase_kernel<<<ntiles, 256, 0, st>>>(ph, d_mats, nmats, d_tiles, iter, sc, s, device_status_ptr());
    return cudaGetLastError();
}

}  // namespace mfsdp
