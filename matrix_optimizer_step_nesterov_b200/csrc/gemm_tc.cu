// tcgen05 / TMEM / TMA engine of the Newton-Schulz GEMM phases (bf16 operands,
// fp32 accumulate) for sm_100a.
//
// One persistent, warp-specialised kernel serves the three phases of an
// iteration (see internal.h for the diagonal-split form they compute):
//   PH_GRAM   C = X X^T      K = c   A: X rows (K-major)   B: X rows (K-major)   upper tiles
//   PH_POLY   C = E_A E_A    K = r   A: E_A rows           B: E_A rows           upper tiles
//   PH_APPLY  C = E_B X      K = r   A: E_B rows           B: X (MN-major)       all tiles
// Output tile 128 x 256 (one cta_group::1 MMA of M=128, N=256, K=16 per 32 B
// of K); K staged 64 deep (one 128-byte swizzle atom of bf16) through a
// 4-stage TMA ring; a double-buffered 2 x 256-column fp32 accumulator in TMEM
// lets the epilogue of one tile overlap the mainloop of the next.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues the MMAs (one elected lane), warps 2-5 run the epilogue, one TMEM
// lane quadrant (32 rows) each.  Every mbarrier wait is bounded: past the
// limit the waiting thread records MFSDP_ERR_TIMEOUT in the device status
// word, raises a CTA-wide abort flag and returns; the other roles see the flag
// in their own waits, the producer drains the loads it has in flight, and
// warp 1 frees TMEM before the CTA exits.
#include "gemm_tc.h"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>
#include <vector>

namespace mfsdp {
namespace {

constexpr int BM = 128;          // tile rows (MMA M)
constexpr int BN = 256;          // tile cols (MMA N)
constexpr int BK = 64;           // K per stage: one 128 B swizzle atom of bf16
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;            // 16 KiB
constexpr int B_BYTES = BN * BK * 2;            // 32 KiB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KiB
constexpr int TMEM_COLS = 2 * BN;               // two fp32 accumulators
constexpr int NUM_THREADS = 192;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align slack*/ + 256 /*barriers*/;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait

// per-matrix TMA descriptors, stored in the workspace head (64-byte aligned)
struct alignas(64) TcMaps {
    CUtensorMap xk[2];   // X bf16 operand, K-major view: dims {c, r}, box {64, 128}
    CUtensorMap xm[2];   // X bf16 operand, MN-major view: dims {c, r}, box {64, 64}
    CUtensorMap ea;      // E_A bf16, dims {r, r}, box {64, 128}
    CUtensorMap eb;      // E_B bf16, dims {r, r}, box {64, 128}
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait.  Returns false when the CTA is aborting (flag raised here on
// timeout, or by another role).
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             int32_t* status) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0u) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                if (status) atomicCAS(status, 0, -6 /* MFSDP_ERR_TIMEOUT */);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
//   K-major operand:  rows 128 B apart, 8-row groups SBO = 1024 B apart (LBO unused).
//   MN-major operand: 64-element MN chunks LBO apart, 8-row K groups SBO = 1024 B apart.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;                 // descriptor version (sm_100)
    d |= 2ull << 61;                 // SWIZZLE_128B
    return d;
}

// Instruction descriptor: D fp32, A/B bf16, A K-major, B K- or MN-major, N=256, M=128.
__host__ __device__ constexpr uint32_t make_idesc(bool b_mn_major) {
    return (1u << 4)                 // D format: F32
         | (1u << 7)                 // A format: BF16
         | (1u << 10)                // B format: BF16
         | ((b_mn_major ? 1u : 0u) << 16)
         | (static_cast<uint32_t>(BN >> 3) << 17)
         | (static_cast<uint32_t>(BM >> 4) << 24);
}

__device__ __forceinline__ void store_bf16(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// ---------------------------------------------------------------------------
// epilogue of one 32-column chunk held by one thread (row gi, columns gj0 + t)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void epilogue_chunk(int ph, const MatDev& md, int iter, const StepScalars& sc,
                                               float sg, int gi, int gj0, int Ncols, const uint32_t (&r)[32]) {
    const int cur = iter & 1, nxt = cur ^ 1;
    if (ph == PH_GRAM) {
        const float s2 = sg * sg;
        #pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int gj = gj0 + t;
            if (gj >= Ncols || gi > gj) continue;
            const float v = s2 * __uint_as_float(r[t]);
            if (gi == gj) {
                md.da[gi] = v;
                md.af[(int64_t)gi * md.lda + gi] = 0.f;
                store_bf16(md.ab + (int64_t)gi * md.lda + gi, 0.f);
            } else {
                md.af[(int64_t)gi * md.lda + gj] = v;
                md.af[(int64_t)gj * md.lda + gi] = v;
                store_bf16(md.ab + (int64_t)gi * md.lda + gj, v);
                store_bf16(md.ab + (int64_t)gj * md.lda + gi, v);
            }
        }
    } else if (ph == PH_POLY) {
        __nv_bfloat16* bm = static_cast<__nv_bfloat16*>(md.bm);
        const float di = md.da[gi];
        #pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int gj = gj0 + t;
            if (gj >= Ncols || gi > gj) continue;
            const float acc = __uint_as_float(r[t]);
            if (gi == gj) {
                md.db[gi] = sc.b * di + sc.c * fmaf(di, di, acc);
                store_bf16(bm + (int64_t)gi * md.lda + gi, 0.f);
            } else {
                const float e = md.af[(int64_t)gi * md.lda + gj];
                const float v = sc.b * e + sc.c * fmaf(di + md.da[gj], e, acc);
                store_bf16(bm + (int64_t)gi * md.lda + gj, v);
                store_bf16(bm + (int64_t)gj * md.lda + gi, v);
            }
        }
    } else {
        const float f = sc.a + md.db[gi];
        float* xrow = md.xf[0] + (int64_t)gi * md.ldx;
        if (ph == PH_APPLY) {
            __nv_bfloat16* xbn = md.xb[nxt] + (int64_t)gi * md.ldx;
            #pragma unroll
            for (int t = 0; t < 32; ++t) {
                const int gj = gj0 + t;
                if (gj >= Ncols) continue;
                const float v = sg * fmaf(f, xrow[gj], __uint_as_float(r[t]));
                xrow[gj] = v;
                store_bf16(xbn + gj, v);
            }
        } else {
            #pragma unroll
            for (int t = 0; t < 32; ++t) {
                const int gj = gj0 + t;
                if (gj >= Ncols) continue;
                const float o = md.shape_scale * (sg * fmaf(f, xrow[gj], __uint_as_float(r[t])));
                const int64_t widx = md.tr ? (int64_t)gj * md.cols + gi : (int64_t)gi * md.cols + gj;
                if (md.update_out) md.update_out[widx] = o;
                if (md.param_bf16) {
                    __nv_bfloat16* w = static_cast<__nv_bfloat16*>(md.param);
                    w[widx] = __float2bfloat16_rn(fmaf(-sc.lr, o, __bfloat162float(w[widx]) * sc.decay));
                } else {
                    float* w = static_cast<float*>(md.param);
                    w[widx] = fmaf(-sc.lr, o, w[widx] * sc.decay);
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// the persistent kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(NUM_THREADS, 1)
tc_phase_kernel(int32_t ph, const MatDev* __restrict__ mats, const TcMaps* __restrict__ maps, int32_t nmats,
                const TileDev* __restrict__ tiles, int32_t ntiles, int32_t iter, StepScalars sc,
                const float* __restrict__ s, int32_t* status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned stage ring (128 B swizzle atoms need 1024 B alignment)
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    // bars: full[STAGES], empty[STAGES], tmem_full[2], tmem_empty[2], mma_done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES);
    const uint32_t tfull0 = smem_u32(bars + 2 * STAGES), tempty0 = smem_u32(bars + 2 * STAGES + 2);
    const uint32_t mma_done = smem_u32(bars + 2 * STAGES + 4);

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(full0 + 8 * i, 1);
            mbar_init(empty0 + 8 * i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(tfull0 + 8 * i, 1);
            mbar_init(tempty0 + 8 * i, 4);   // one arrive per epilogue warp
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const bool gemm = (ph == PH_APPLY || ph == PH_FINAL);
    const int cur = iter & 1;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int issued[STAGES];                  // parity of the last fill issued per stage, -1 = none
            #pragma unroll
            for (int i = 0; i < STAGES; ++i) issued[i] = -1;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                const TileDev td = tiles[t];
                const MatDev& md = mats[td.mat];
                const TcMaps& mp = maps[td.mat];
                const int K = (ph == PH_GRAM) ? md.c : md.r;
                const int nk = (K + BK - 1) / BK;
                const CUtensorMap* amap = (ph == PH_GRAM) ? &mp.xk[cur] : (ph == PH_POLY) ? &mp.ea : &mp.eb;
                const CUtensorMap* bmap = (ph == PH_GRAM) ? &mp.xk[cur] : (ph == PH_POLY) ? &mp.ea : &mp.xm[cur];
                const int i0 = td.tm * BM, j0 = td.tn * BN;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!wait_bounded(empty0 + 8 * stage, phase ^ 1, abort_flag, status)) { ok = false; break; }
                    const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
                    const uint32_t fb = full0 + 8 * stage;
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(sa, amap, fb, kb * BK, i0);
                    if (!gemm) {
                        tma_load_2d(sb, bmap, fb, kb * BK, j0);
                        tma_load_2d(sb + BN / 2 * BK * 2, bmap, fb, kb * BK, j0 + BN / 2);
                    } else {
                        #pragma unroll
                        for (int q = 0; q < BN / 64; ++q)
                            tma_load_2d(sb + q * (BK * 128), bmap, fb, j0 + 64 * q, kb * BK);
                    }
                    issued[stage] = static_cast<int>(phase);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                // aborting: wait (bounded, 10 ms each) until every issued load has landed
                for (int i = 0; i < STAGES; ++i) {
                    if (issued[i] < 0) continue;
                    const unsigned long long t0 = globaltimer();
                    while (!mbar_try_wait(full0 + 8 * i, static_cast<uint32_t>(issued[i])) &&
                           globaltimer() - t0 < 10000000ull) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = make_idesc(gemm);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                const TileDev td = tiles[t];
                const MatDev& md = mats[td.mat];
                const int K = (ph == PH_GRAM) ? md.c : md.r;
                const int nk = (K + BK - 1) / BK;
                if (!wait_bounded(tempty0 + 8 * acc, acc_phase ^ 1, abort_flag, status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!wait_bounded(full0 + 8 * stage, phase, abort_flag, status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
                    #pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t ad = smem_desc(sa + kk * 32, 16, 1024);
                        const uint64_t bd = gemm ? smem_desc(sb + kk * 16 * 128, BK * 128, 1024)
                                                 : smem_desc(sb + kk * 32, 16, 1024);
                        tc_mma(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(empty0 + 8 * stage);     // stage free once these MMAs finish
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                tc_commit(tfull0 + 8 * acc);           // accumulator ready for the epilogue
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
            // every MMA this thread issued has completed before TMEM is freed (bounded)
            tc_commit(mma_done);
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(mma_done, 0) && globaltimer() - t0 < 100000000ull) {
            }
        }
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            const TileDev td = tiles[t];
            const MatDev& md = mats[td.mat];
            const int Mrows = md.r;
            const int Ncols = gemm ? md.c : md.r;
            bool ok = true;
            if (lane == 0) ok = wait_bounded(tfull0 + 8 * acc, acc_phase, abort_flag, status);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            tc_fence_after();
            const float sg = (iter == 0) ? s[td.mat] : 1.0f;
            const int gi = td.tm * BM + quad * 32 + lane;
            const uint32_t trow = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * BN;
            // skip whole chunks that lie left of the diagonal in symmetric phases
            #pragma unroll 1
            for (int q = 0; q < BN / 32; ++q) {
                const int gj0 = td.tn * BN + q * 32;
                uint32_t r[32];
                tmem_ld32(trow + q * 32, r);       // warp-collective: every lane executes it
                if (gi < Mrows && gj0 < Ncols) epilogue_chunk(ph, md, iter, sc, sg, gi, gj0, Ncols, r);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

bool encode_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld_elems,
               uint32_t box_inner, uint32_t box_outer) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {ld_elems * 2};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_available() { return true; }

size_t tc_maps_bytes(size_t nmats) { return nmats * sizeof(TcMaps); }

bool tc_encode_maps(const std::vector<MatDev>& mats, void* host_out) {
    TcMaps* out = static_cast<TcMaps*>(host_out);
    for (size_t i = 0; i < mats.size(); ++i) {
        const MatDev& m = mats[i];
        TcMaps& mp = out[i];
        for (int b = 0; b < 2; ++b) {
            if (!encode_2d(&mp.xk[b], m.xb[b], m.c, m.r, m.ldx, BK, BM)) return false;
            if (!encode_2d(&mp.xm[b], m.xb[b], m.c, m.r, m.ldx, 64, BK)) return false;
        }
        if (!encode_2d(&mp.ea, m.ab, m.r, m.r, m.lda, BK, BM)) return false;
        if (!encode_2d(&mp.eb, m.bm, m.r, m.r, m.lda, BK, BM)) return false;
    }
    return true;
}

void tc_build_tiles(const std::vector<MatDev>& mats, std::vector<TileDev>& gram, std::vector<TileDev>& poly,
                    std::vector<TileDev>& gen) {
    for (int32_t mi = 0; mi < static_cast<int32_t>(mats.size()); ++mi) {
        const MatDev& m = mats[mi];
        const int tm_n = (m.r + BM - 1) / BM;
        const int tn_sym = (m.r + BN - 1) / BN;
        const int tn_gen = (m.c + BN - 1) / BN;
        for (int i = 0; i < tm_n; ++i) {
            for (int j = 0; j < tn_sym; ++j) {
                // keep tiles that reach the upper triangle (row i*BM <= last column of the tile)
                if (i * BM > j * BN + BN - 1) continue;
                gram.push_back({mi, i, j, (m.c + BK - 1) / BK});
                poly.push_back({mi, i, j, (m.r + BK - 1) / BK});
            }
            for (int j = 0; j < tn_gen; ++j) gen.push_back({mi, i, j, (m.r + BK - 1) / BK});
        }
    }
    // longest first; ties keep a matrix's tiles together (L2 reuse of its operands)
    auto lpt = [](const TileDev& a, const TileDev& b) {
        if (a.kblk != b.kblk) return a.kblk > b.kblk;
        if (a.mat != b.mat) return a.mat < b.mat;
        if (a.tm != b.tm) return a.tm < b.tm;
        return a.tn < b.tn;
    };
    std::stable_sort(gram.begin(), gram.end(), lpt);
    std::stable_sort(poly.begin(), poly.end(), lpt);
    std::stable_sort(gen.begin(), gen.end(), lpt);
}

cudaError_t launch_gemm_tc(Phase ph, const MatDev* d_mats, const void* d_maps, int32_t nmats,
                           const TileDev* d_tiles, int32_t ntiles, int32_t iter, const StepScalars& sc,
                           const float* s, cudaStream_t st) {
    if (ntiles <= 0) return cudaSuccess;
    static int sms = 0;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(tc_phase_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
        attr_set = true;
    }
    const int grid = std::min(ntiles, sms);
    tc_phase_kernel<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(ph, d_mats, static_cast<const TcMaps*>(d_maps), nmats,
                                                           d_tiles, ntiles, iter, sc, s, device_status_ptr());
    return cudaGetLastError();
}

}  // namespace mfsdp
