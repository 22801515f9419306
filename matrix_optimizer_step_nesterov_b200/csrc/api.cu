// C ABI entry points of libmfsdp: argument validation, the workspace layout,
// the grouped tile tables and the launch sequence of the owner-local step.
//
// Step (per matrix, grouped over the owner's matrix list): "MatrixFSDP:
// communication-free matrix optimizers under ZeRO-3 parameter sharding",
// arxivlens summary page, Abstract -- the owner holds the whole matrix and
// runs Muon's momentum + Newton-Schulz update locally; the tail stays on AdamW.
#include "../../include/mfsdp.h"
#include "internal.h"
#include "gemm_tc.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <atomic>
#include <mutex>
#include <unordered_map>
#include <vector>

namespace mfsdp {
namespace {

constexpr size_t kAlign = 256;
constexpr size_t kRegionSlack = 128;

size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }
int64_t round8(int64_t x) { return (x + 7) / 8 * 8; }

int check_device() {
    static std::atomic<int> cached[64];  // 0 unknown, 1 ok, -1 unsupported (zero-initialised)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MFSDP_ERR_CUDA;
    }
    if (dev < 0 || dev >= 64) return MFSDP_ERR_UNSUPPORTED_DEVICE;
    if (cached[dev].load(std::memory_order_relaxed) == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            cudaGetLastError();
            return MFSDP_ERR_CUDA;
        }
        cached[dev].store((major == 10 && minor == 0) ? 1 : -1, std::memory_order_relaxed);
    }
    return cached[dev].load(std::memory_order_relaxed) == 1 ? MFSDP_OK : MFSDP_ERR_UNSUPPORTED_DEVICE;
}

bool aligned(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

int validate_hparams(const mfsdp_muon_hparams* hp) {
    if (!hp) return MFSDP_ERR_INVALID_ARG;
    if (hp->mode != MFSDP_MODE_FP32 && hp->mode != MFSDP_MODE_BF16) return MFSDP_ERR_INVALID_ARG;
    if (hp->ns_steps < 0 || hp->ns_steps > 16) return MFSDP_ERR_INVALID_ARG;
    if (hp->nesterov != 0 && hp->nesterov != 1) return MFSDP_ERR_INVALID_ARG;
    if (!std::isfinite(hp->lr) || !std::isfinite(hp->beta) || !std::isfinite(hp->weight_decay) ||
        !std::isfinite(hp->eps) || !std::isfinite(hp->a) || !std::isfinite(hp->b) || !std::isfinite(hp->c))
        return MFSDP_ERR_INVALID_ARG;
    if (hp->eps < 0.f) return MFSDP_ERR_INVALID_ARG;
    return MFSDP_OK;
}

int validate_matrix(const mfsdp_matrix& m, const mfsdp_owner_segments* seg) {
    if (m.rows < 0 || m.cols < 0) return MFSDP_ERR_INVALID_ARG;
    if (m.rows > (1LL << 30) || m.cols > (1LL << 30)) return MFSDP_ERR_INVALID_ARG;
    if (m.param_dtype != MFSDP_DTYPE_F32 && m.param_dtype != MFSDP_DTYPE_BF16) return MFSDP_ERR_UNSUPPORTED_DTYPE;
    if (m.grad_dtype != MFSDP_DTYPE_F32 && m.grad_dtype != MFSDP_DTYPE_BF16) return MFSDP_ERR_UNSUPPORTED_DTYPE;
    if (m.rows == 0 || m.cols == 0) return MFSDP_OK;
    if (!m.param || !m.momentum) return MFSDP_ERR_INVALID_ARG;
    const size_t pe = m.param_dtype == MFSDP_DTYPE_BF16 ? 2 : 4;
    const size_t ge = m.grad_dtype == MFSDP_DTYPE_BF16 ? 2 : 4;
    if (!aligned(m.param, pe)) return MFSDP_ERR_MISALIGNED;
    if (seg) {
        if (seg->nparts < 1 || seg->nparts > MFSDP_MAX_PARTS || !seg->grad_parts) return MFSDP_ERR_INVALID_ARG;
        if (seg->ncopies < 0 || seg->ncopies > MFSDP_MAX_COPIES) return MFSDP_ERR_INVALID_ARG;
        if (seg->ncopies > 0 && !seg->param_copies) return MFSDP_ERR_INVALID_ARG;
        for (int32_t r = 0; r < seg->nparts; ++r) {
            if (!seg->grad_parts[r]) return MFSDP_ERR_INVALID_ARG;
            if (!aligned(seg->grad_parts[r], ge)) return MFSDP_ERR_MISALIGNED;
        }
        for (int32_t d = 0; d < seg->ncopies; ++d) {
            if (!seg->param_copies[d]) return MFSDP_ERR_INVALID_ARG;
            if (!aligned(seg->param_copies[d], pe)) return MFSDP_ERR_MISALIGNED;
        }
    } else {
        if (!m.grad) return MFSDP_ERR_INVALID_ARG;
        if (!aligned(m.grad, ge)) return MFSDP_ERR_MISALIGNED;
    }
    if (!aligned(m.momentum, 4)) return MFSDP_ERR_MISALIGNED;
    if (m.update_out && !aligned(m.update_out, 4)) return MFSDP_ERR_MISALIGNED;
    return MFSDP_OK;
}

// [begin, end) byte ranges of every user buffer, to reject aliasing between matrices
int check_no_alias(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n) {
    struct Range { uintptr_t b, e; int32_t owner; bool writable; };
    std::vector<Range> rs;
    rs.reserve(static_cast<size_t>(n) * 4);
    for (int32_t i = 0; i < n; ++i) {
        const mfsdp_matrix& m = mats[i];
        if (m.rows == 0 || m.cols == 0) continue;
        const uintptr_t numel = static_cast<uintptr_t>(m.rows * m.cols);
        const uintptr_t pe = m.param_dtype == MFSDP_DTYPE_BF16 ? 2 : 4;
        const uintptr_t ge = m.grad_dtype == MFSDP_DTYPE_BF16 ? 2 : 4;
        rs.push_back({reinterpret_cast<uintptr_t>(m.param), reinterpret_cast<uintptr_t>(m.param) + numel * pe, i, true});
        if (!segs)
            rs.push_back({reinterpret_cast<uintptr_t>(m.grad), reinterpret_cast<uintptr_t>(m.grad) + numel * ge, i, false});
        rs.push_back({reinterpret_cast<uintptr_t>(m.momentum), reinterpret_cast<uintptr_t>(m.momentum) + numel * 4, i, true});
        if (m.update_out)
            rs.push_back({reinterpret_cast<uintptr_t>(m.update_out), reinterpret_cast<uintptr_t>(m.update_out) + numel * 4, i, true});
    }
    std::sort(rs.begin(), rs.end(), [](const Range& x, const Range& y) { return x.b < y.b; });
    // any overlap that involves a written range is an error (two grads may share memory)
    uintptr_t max_end_w = 0, max_end_any = 0;
    for (const Range& r : rs) {
        if (r.b < max_end_w) return MFSDP_ERR_INVALID_ARG;
        if (r.writable && r.b < max_end_any) return MFSDP_ERR_INVALID_ARG;
        max_end_any = std::max(max_end_any, r.e);
        if (r.writable) max_end_w = std::max(max_end_w, r.e);
    }
    return MFSDP_OK;
}

// The GEMM engine of each mode: bf16 operands run on the tcgen05 tensor cores,
// fp32 mode (no tf32) on the FFMA pipes.  There is no fallback between them.
enum class Engine { Simt, Tc };

Engine pick_engine(const mfsdp_muon_hparams* hp) {
    return hp->mode == MFSDP_MODE_BF16 ? Engine::Tc : Engine::Simt;
}

// Workspace plan: head (descriptor table, tile tables, partials, scales), then
// per-matrix X / A / B buffers, every region 256-byte aligned.
struct Layout {
    std::vector<MatDev> mats;          // device records (workspace pointers filled if base given)
    std::vector<TileDev> sym_tiles;    // PH_GRAM
    std::vector<TileDev> poly_tiles;   // PH_POLY
    std::vector<TileDev> gen_tiles;    // PH_APPLY / PH_FINAL
    // tensor-core engine: each table partitioned over its launch's clusters
    // (segment offsets, clusters + 1 entries, in a fixed-size head slot)
    std::vector<int32_t> sym_seg, poly_seg, gen_seg;
    std::vector<uint64_t> ptrs;        // owner-segment part and copy pointers, per matrix
    size_t off_ptrs = 0;
    int32_t mom_tiles = 0;
    int32_t mom_groups = 0;            // groups of the streaming kernels, flat ones first
    int32_t flat_groups = 0;           // groups of the flat matrices: [0, flat_groups)
    size_t off_mats = 0, off_maps = 0, off_sym = 0, off_poly = 0, off_gen = 0, off_partials = 0, off_s = 0;
    size_t off_sym_seg = 0, off_poly_seg = 0, off_gen_seg = 0;
    size_t head_end = 0, maps_bytes = 0;
    size_t total = 0;
    Engine engine = Engine::Simt;
};

// Clusters a persistent phase may use at most; the head reserves room for
// that many segment offsets per phase, so the layout does not depend on the
// device.
constexpr int kMaxClusters = 1024;

void build_tiles(Layout& L, Engine eng, int max_clusters) {
    L.sym_tiles.clear();
    L.poly_tiles.clear();
    L.gen_tiles.clear();
    L.sym_seg.clear();
    L.poly_seg.clear();
    L.gen_seg.clear();
    if (eng == Engine::Tc) {
        tc_build_tiles(L.mats, std::max(1, std::min(max_clusters, kMaxClusters)), L.sym_tiles, L.poly_tiles,
                       L.gen_tiles, L.sym_seg, L.poly_seg, L.gen_seg);
        return;
    }
    const int T = kSimtTile;
    for (int32_t mi = 0; mi < static_cast<int32_t>(L.mats.size()); ++mi) {
        const MatDev& m = L.mats[mi];
        const int tr_ = (m.r + T - 1) / T, tc_ = (m.c + T - 1) / T;
        for (int i = 0; i < tr_; ++i)
            for (int j = i; j < tr_; ++j) L.sym_tiles.push_back({mi, i, j, (m.c + 7) / 8});
        for (int i = 0; i < tr_; ++i)
            for (int j = 0; j < tc_; ++j) L.gen_tiles.push_back({mi, i, j, (m.r + 7) / 8});
    }
    L.poly_tiles = L.sym_tiles;
}

// Self-check of the host-built tile tables: every output tile of every matrix
// appears exactly once - all tiles of X for the general phase, the tiles that
// reach the upper triangle of the r x r result for GRAM and POLY - with a
// positive K depth.  A failure is a bug in the tile builder, never the caller's.
bool tiles_cover(const Layout& L, int tm_edge, int tn_edge) {
    const int32_t nm = static_cast<int32_t>(L.mats.size());
    auto check = [&](const std::vector<TileDev>& tiles, bool sym) {
        std::vector<size_t> base(static_cast<size_t>(nm) + 1, 0);
        std::vector<int> ncols(static_cast<size_t>(nm), 0), nrows(static_cast<size_t>(nm), 0);
        for (int32_t i = 0; i < nm; ++i) {
            const MatDev& m = L.mats[i];
            nrows[i] = (m.r + tm_edge - 1) / tm_edge;
            ncols[i] = ((sym ? m.r : m.c) + tn_edge - 1) / tn_edge;
            base[i + 1] = base[i] + static_cast<size_t>(nrows[i]) * ncols[i];
        }
        std::vector<uint8_t> seen(base[nm], 0);
        for (const TileDev& t : tiles) {
            if (t.mat < 0 || t.mat >= nm || t.kblk <= 0) return false;
            if (t.tm < 0 || t.tm >= nrows[t.mat] || t.tn < 0 || t.tn >= ncols[t.mat]) return false;
            if (sym && static_cast<int64_t>(t.tm) * tm_edge > static_cast<int64_t>(t.tn) * tn_edge + tn_edge - 1)
                return false;
            uint8_t& c = seen[base[t.mat] + static_cast<size_t>(t.tm) * ncols[t.mat] + t.tn];
            if (c) return false;
            c = 1;
        }
        for (int32_t i = 0; i < nm; ++i)
            for (int a = 0; a < nrows[i]; ++a)
                for (int b = 0; b < ncols[i]; ++b) {
                    const bool wanted = !sym || static_cast<int64_t>(a) * tm_edge <= static_cast<int64_t>(b) * tn_edge + tn_edge - 1;
                    if (seen[base[i] + static_cast<size_t>(a) * ncols[i] + b] != (wanted ? 1 : 0)) return false;
                }
        return true;
    };
    // segments: clusters + 1 nondecreasing offsets from 0 to the table's size
    auto segs_ok = [](const std::vector<int32_t>& seg, size_t ntiles) {
        if (seg.size() < 2 || seg.size() > static_cast<size_t>(kMaxClusters) + 1) return false;
        if (seg.front() != 0 || static_cast<size_t>(seg.back()) != ntiles) return false;
        for (size_t k = 1; k < seg.size(); ++k)
            if (seg[k] < seg[k - 1]) return false;
        return true;
    };
    if (L.engine == Engine::Tc &&
        !(segs_ok(L.sym_seg, L.sym_tiles.size()) && segs_ok(L.poly_seg, L.poly_tiles.size()) &&
          segs_ok(L.gen_seg, L.gen_tiles.size())))
        return false;
    return check(L.sym_tiles, true) && check(L.poly_tiles, true) && check(L.gen_tiles, false);
}

// max_clusters: the tensor-core engine's persistent grid on this device (any
// value >= 1 when only the size is wanted: it changes no offset)
int build_layout(const mfsdp_matrix* in, const mfsdp_owner_segments* segs, int32_t n,
                 const mfsdp_muon_hparams* hp, char* base, Layout& L, int max_clusters) {
    const bool bf16 = hp->mode == MFSDP_MODE_BF16;
    L.engine = pick_engine(hp);
    L.mats.clear();
    L.ptrs.clear();
    std::vector<size_t> ptr_first;     // index into L.ptrs of each live matrix's part pointers
    int32_t tile0 = 0, grp0 = 0;
    for (int32_t i = 0; i < n; ++i) {
        const mfsdp_matrix& u = in[i];
        if (u.rows == 0 || u.cols == 0) continue;
        MatDev m{};
        bool vec_parts = true, vec_parts16 = true;
        if (segs) {
            const mfsdp_owner_segments& sg = segs[i];
            m.nparts = sg.nparts;
            m.ncopies = sg.ncopies;
            ptr_first.push_back(L.ptrs.size());
            for (int32_t r = 0; r < sg.nparts; ++r) {
                L.ptrs.push_back(reinterpret_cast<uint64_t>(sg.grad_parts[r]));
                vec_parts = vec_parts && aligned(sg.grad_parts[r], u.grad_dtype == MFSDP_DTYPE_BF16 ? 8 : 16);
                vec_parts16 = vec_parts16 && aligned(sg.grad_parts[r], 16);
            }
            for (int32_t d = 0; d < sg.ncopies; ++d) L.ptrs.push_back(reinterpret_cast<uint64_t>(sg.param_copies[d]));
        } else {
            ptr_first.push_back(L.ptrs.size());
        }
        m.param = u.param;
        m.grad = u.grad;
        m.buf = u.momentum;
        m.update_out = u.update_out;
        m.rows = u.rows;
        m.cols = u.cols;
        m.tr = u.rows > u.cols ? 1 : 0;
        m.r = static_cast<int32_t>(std::min(u.rows, u.cols));
        m.c = static_cast<int32_t>(std::max(u.rows, u.cols));
        m.ldx = round8(m.c);
        m.lda = round8(m.r);
        m.param_bf16 = u.param_dtype == MFSDP_DTYPE_BF16;
        m.grad_bf16 = u.grad_dtype == MFSDP_DTYPE_BF16;
        m.mom_tiles_n = static_cast<int32_t>((u.cols + kMomTile - 1) / kMomTile);
        const int64_t tiles = ((u.rows + kMomTile - 1) / kMomTile) * m.mom_tiles_n;
        if (tile0 + tiles > (1LL << 31) - 1) return MFSDP_ERR_INVALID_ARG;
        tile0 += static_cast<int32_t>(tiles);
        m.mom_vec = (u.cols % 4 == 0) && aligned(u.momentum, 16) &&
                    (segs ? vec_parts : aligned(u.grad, u.grad_dtype == MFSDP_DTYPE_BF16 ? 8 : 16));
        // flat runs: X = M (no transpose) with ldx == cols, and every access 16 bytes wide
        bool flat = u.rows <= u.cols && u.cols % 8 == 0 && aligned(u.momentum, 16) && aligned(u.param, 16) &&
                    (!u.update_out || aligned(u.update_out, 16)) && (segs ? vec_parts16 : aligned(u.grad, 16));
        if (segs)
            for (int32_t d = 0; d < segs[i].ncopies; ++d) flat = flat && aligned(segs[i].param_copies[d], 16);
        m.mom_flat = flat ? 1 : 0;
        const int64_t groups = flat ? (u.rows * u.cols + kFlatGroup - 1) / kFlatGroup
                                    : (tiles + kMomGroup - 1) / kMomGroup;
        if (grp0 + groups > (1LL << 31) - 1) return MFSDP_ERR_INVALID_ARG;
        m.mom_groups_n = static_cast<int32_t>(groups);
        grp0 += static_cast<int32_t>(groups);
        m.shape_scale = static_cast<float>(std::sqrt(std::max(1.0, static_cast<double>(u.rows) / u.cols)));
        L.mats.push_back(m);
    }
    // The streaming kernels run the flat matrices' groups and the tiled ones' in
    // separate launches: order the records flat first (stable), then number the
    // groups in that order, so that each launch covers one contiguous range.
    {
        std::vector<size_t> order(L.mats.size());
        for (size_t k = 0; k < order.size(); ++k) order[k] = k;
        std::stable_partition(order.begin(), order.end(), [&](size_t k) { return L.mats[k].mom_flat != 0; });
        std::vector<MatDev> mats;
        std::vector<size_t> firsts;
        mats.reserve(order.size());
        firsts.reserve(order.size());
        for (size_t k : order) {
            mats.push_back(L.mats[k]);
            firsts.push_back(ptr_first[k]);
        }
        L.mats.swap(mats);
        ptr_first.swap(firsts);
        int32_t g = 0;
        L.flat_groups = 0;
        for (MatDev& m : L.mats) {
            m.mom_grp0 = g;
            g += m.mom_groups_n;
            if (m.mom_flat) L.flat_groups = g;
        }
    }
    L.mom_tiles = tile0;
    L.mom_groups = grp0;
    build_tiles(L, L.engine, max_clusters);
    if (L.engine == Engine::Tc ? !tiles_cover(L, tc_tile_rows(), tc_tile_cols())
                               : !tiles_cover(L, kSimtTile, kSimtTile))
        return MFSDP_ERR_INVALID_ARG;
    const size_t nm = L.mats.size();
    size_t off = 0;
    L.off_mats = off;      off = align_up(off + nm * sizeof(MatDev));
    L.off_ptrs = off;      off = align_up(off + L.ptrs.size() * sizeof(uint64_t));
    for (size_t k = 0; k < nm; ++k) {
        MatDev& m = L.mats[k];
        const uint64_t* first = reinterpret_cast<const uint64_t*>(base ? base + L.off_ptrs : nullptr) + ptr_first[k];
        m.gparts = m.nparts ? reinterpret_cast<const void* const*>(first) : nullptr;
        m.pcopies = m.ncopies ? reinterpret_cast<void* const*>(first + m.nparts) : nullptr;
    }
    L.maps_bytes = L.engine == Engine::Tc ? tc_maps_bytes(nm) : 0;
    L.off_maps = off;      off = align_up(off + L.maps_bytes);
    L.off_sym = off;       off = align_up(off + L.sym_tiles.size() * sizeof(TileDev));
    L.off_poly = off;      off = align_up(off + L.poly_tiles.size() * sizeof(TileDev));
    L.off_gen = off;       off = align_up(off + L.gen_tiles.size() * sizeof(TileDev));
    const size_t seg_bytes = L.engine == Engine::Tc ? (kMaxClusters + 1) * sizeof(int32_t) : 0;
    L.off_sym_seg = off;   off = align_up(off + seg_bytes);
    L.off_poly_seg = off;  off = align_up(off + seg_bytes);
    L.off_gen_seg = off;   off = align_up(off + seg_bytes);
    L.off_partials = off;  off = align_up(off + static_cast<size_t>(L.mom_groups) * sizeof(float));
    L.off_s = off;         off = align_up(off + nm * sizeof(float));
    L.head_end = off;
    for (MatDev& m : L.mats) {
        const size_t x_elems = static_cast<size_t>(m.r) * m.ldx;
        const size_t a_elems = static_cast<size_t>(m.r) * m.lda;
        // every region keeps at least kRegionSlack bytes after its end: a tensor-core
        // operand load may read up to 126 bytes past a matrix's last valid element
        // (values that only reach output columns the epilogue discards)
        auto take = [&](size_t bytes) -> char* {
            char* p = base ? base + off : nullptr;
            off = align_up(off + bytes + kRegionSlack);
            return p;
        };
        if (bf16) {
            m.xf[0] = m.xf[1] = nullptr;
            m.xb[0] = reinterpret_cast<__nv_bfloat16*>(take(x_elems * 2));
            m.xb[1] = reinterpret_cast<__nv_bfloat16*>(take(x_elems * 2));
            m.xlo[0] = reinterpret_cast<__nv_bfloat16*>(take(x_elems * 2));
            m.xlo[1] = reinterpret_cast<__nv_bfloat16*>(take(x_elems * 2));
            m.af = nullptr;
            m.ab = reinterpret_cast<__nv_bfloat16*>(take(a_elems * 2));
            m.bm = take(a_elems * 2);
            m.da = reinterpret_cast<float*>(take(static_cast<size_t>(m.r) * 4));
            m.db = reinterpret_cast<float*>(take(static_cast<size_t>(m.r) * 4));
        } else {
            m.xf[0] = reinterpret_cast<float*>(take(x_elems * 4));
            m.xf[1] = reinterpret_cast<float*>(take(x_elems * 4));
            m.xb[0] = m.xb[1] = nullptr;
            m.xlo[0] = m.xlo[1] = nullptr;
            m.af = reinterpret_cast<float*>(take(a_elems * 4));
            m.ab = nullptr;
            m.bm = take(a_elems * 4);
            m.da = reinterpret_cast<float*>(take(static_cast<size_t>(m.r) * 4));
            m.db = reinterpret_cast<float*>(take(static_cast<size_t>(m.r) * 4));
        }
    }
    L.total = off;
    return MFSDP_OK;
}

// host cache: the head bytes last uploaded into each workspace
struct CacheEntry { int dev; std::vector<char> head; };
std::mutex g_cache_mu;
std::unordered_map<uintptr_t, CacheEntry> g_cache;

int validate_all(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n,
                 const mfsdp_muon_hparams* hp) {
    if (n < 0) return MFSDP_ERR_INVALID_ARG;
    int st = validate_hparams(hp);
    if (st) return st;
    if (n > 0 && !mats) return MFSDP_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n; ++i) {
        st = validate_matrix(mats[i], segs ? &segs[i] : nullptr);
        if (st) return st;
    }
    return check_no_alias(mats, segs, n);
}

int workspace_size_impl(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n,
                        const mfsdp_muon_hparams* hp, size_t* bytes) {
    if (!bytes) return MFSDP_ERR_INVALID_ARG;
    int st = validate_all(mats, segs, n, hp);
    if (st) return st;
    Layout L;
    st = build_layout(mats, segs, n, hp, nullptr, L, 1);
    if (st) return st;
    *bytes = L.mats.empty() ? 0 : L.total;
    return MFSDP_OK;
}

}  // namespace

}  // namespace mfsdp

using namespace mfsdp;

extern "C" int mfsdp_muon_workspace_size(const mfsdp_matrix* mats, int32_t n, const mfsdp_muon_hparams* hp,
                                         size_t* bytes) {
    return workspace_size_impl(mats, nullptr, n, hp, bytes);
}

extern "C" int mfsdp_muon_workspace_size_p2p(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n,
                                             const mfsdp_muon_hparams* hp, size_t* bytes) {
    if (n > 0 && !segs) return MFSDP_ERR_INVALID_ARG;
    return workspace_size_impl(mats, segs, n, hp, bytes);
}

extern "C" int mfsdp_muon_step_launches(const mfsdp_matrix* mats, int32_t n, const mfsdp_muon_hparams* hp,
                                        int32_t* launches) {
    if (!launches) return MFSDP_ERR_INVALID_ARG;
    int st = validate_all(mats, nullptr, n, hp);
    if (st) return st;
    Layout L;
    st = build_layout(mats, nullptr, n, hp, nullptr, L, 1);
    if (st) return st;
    if (L.mats.empty()) {
        *launches = 0;
        return MFSDP_OK;
    }
    // momentum and parameter write: one launch each for the flat and the tiled matrices present
    const int32_t streaming = (L.flat_groups > 0 ? 1 : 0) + (L.mom_groups > L.flat_groups ? 1 : 0);
    *launches = 2 * streaming + 1 + 3 * hp->ns_steps;
    return MFSDP_OK;
}

extern "C" int mfsdp_muon_forget_workspace(void* workspace) {
    std::lock_guard<std::mutex> lock(g_cache_mu);
    g_cache.erase(reinterpret_cast<uintptr_t>(workspace));
    return MFSDP_OK;
}

extern "C" int mfsdp_muon_forget_workspace_range(void* workspace, size_t bytes) {
    const uintptr_t b = reinterpret_cast<uintptr_t>(workspace), e = b + bytes;
    if (e < b) return MFSDP_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_cache_mu);
    for (auto it = g_cache.begin(); it != g_cache.end();) {
        if (it->first >= b && it->first < e) it = g_cache.erase(it);
        else ++it;
    }
    return MFSDP_OK;
}

extern "C" int mfsdp_muon_step(const mfsdp_matrix* mats, int32_t n, const mfsdp_muon_hparams* hp,
                               void* workspace, size_t workspace_bytes, void* stream) {
    return muon_step_impl(mats, nullptr, n, hp, workspace, workspace_bytes, stream);
}

extern "C" int mfsdp_muon_step_p2p(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n,
                                   const mfsdp_muon_hparams* hp, void* workspace, size_t workspace_bytes,
                                   void* stream) {
    if (n > 0 && !segs) return MFSDP_ERR_INVALID_ARG;
    return muon_step_impl(mats, segs, n, hp, workspace, workspace_bytes, stream);
}

namespace {

constexpr int32_t kMaxOverlapGroups = 64;

// Contiguous groups of about equal Newton-Schulz work, in list order: group k
// ends at the first matrix where the running dense FLOP count reaches (k + 1) / G
// of the total.  Returns G + 1 boundaries (empty groups dropped).
std::vector<int32_t> overlap_bounds(const mfsdp_matrix* mats, int32_t n, int32_t groups) {
    std::vector<double> cost(static_cast<size_t>(n), 0.0);
    double total = 0.0;
    for (int32_t i = 0; i < n; ++i) {
        const double r = static_cast<double>(std::min(mats[i].rows, mats[i].cols));
        const double c = static_cast<double>(std::max(mats[i].rows, mats[i].cols));
        cost[i] = 4.0 * r * r * c + 2.0 * r * r * r;
        total += cost[i];
    }
    std::vector<int32_t> b{0};
    double acc = 0.0;
    int32_t k = 1;
    for (int32_t i = 0; i < n; ++i) {
        acc += cost[i];
        if (k < groups && acc >= total * k / groups && i + 1 < n) {
            b.push_back(i + 1);
            while (k < groups && acc >= total * k / groups) ++k;
        }
    }
    b.push_back(n);
    return b;
}

// The owner segments of one group with the copies left out (the copies of the
// overlapped form move on the copy engines instead).
std::vector<mfsdp_owner_segments> segs_without_copies(const mfsdp_owner_segments* segs, int32_t b0, int32_t b1) {
    std::vector<mfsdp_owner_segments> out(segs + b0, segs + b1);
    for (mfsdp_owner_segments& s : out) {
        s.param_copies = nullptr;
        s.ncopies = 0;
    }
    return out;
}

// Per-group workspace offsets (256-byte aligned) and the total.
int overlap_workspace(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n,
                      const mfsdp_muon_hparams* hp, const std::vector<int32_t>& b, std::vector<size_t>& off,
                      std::vector<size_t>& bytes, size_t* total) {
    off.clear();
    bytes.clear();
    size_t t = 0;
    for (size_t g = 0; g + 1 < b.size(); ++g) {
        const std::vector<mfsdp_owner_segments> gs = segs_without_copies(segs, b[g], b[g + 1]);
        size_t sz = 0;
        const int st = workspace_size_impl(mats + b[g], gs.data(), b[g + 1] - b[g], hp, &sz);
        if (st) return st;
        off.push_back(t);
        bytes.push_back(sz);
        t = align_up(t + sz);
    }
    *total = t;
    return MFSDP_OK;
}

}  // namespace

extern "C" int mfsdp_muon_workspace_size_p2p_overlap(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs,
                                                     int32_t n, const mfsdp_muon_hparams* hp, int32_t groups,
                                                     size_t* bytes) {
    if (!bytes || groups < 1 || groups > kMaxOverlapGroups || (n > 0 && !segs)) return MFSDP_ERR_INVALID_ARG;
    int st = validate_all(mats, segs, n, hp);
    if (st) return st;
    std::vector<size_t> off, sz;
    return overlap_workspace(mats, segs, n, hp, overlap_bounds(mats, n, groups), off, sz, bytes);
}

extern "C" int mfsdp_muon_step_p2p_overlap(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n,
                                           const mfsdp_muon_hparams* hp, int32_t groups, void* workspace,
                                           size_t workspace_bytes, void* stream, void* copy_stream) {
    if (groups < 1 || groups > kMaxOverlapGroups || (n > 0 && !segs)) return MFSDP_ERR_INVALID_ARG;
    int st = validate_all(mats, segs, n, hp);
    if (st) return st;
    const std::vector<int32_t> b = overlap_bounds(mats, n, groups);
    std::vector<size_t> off, sz;
    size_t total = 0;
    st = overlap_workspace(mats, segs, n, hp, b, off, sz, &total);
    if (st) return st;
    if (total == 0) return MFSDP_OK;
    if (!workspace) return MFSDP_ERR_INVALID_ARG;
    if (!aligned(workspace, kAlign)) return MFSDP_ERR_MISALIGNED;
    if (workspace_bytes < total) return MFSDP_ERR_WORKSPACE_TOO_SMALL;
    st = check_device();
    if (st) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream), cs = static_cast<cudaStream_t>(copy_stream);
    const size_t ngroups = b.size() - 1;
    std::vector<cudaEvent_t> ev(ngroups + 1, nullptr);
    auto release = [&]() {
        for (cudaEvent_t e : ev)
            if (e) cudaEventDestroy(e);   // released once the recorded work completes
    };
    for (cudaEvent_t& e : ev) {
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
            cudaGetLastError();
            release();
            return MFSDP_ERR_CUDA;
        }
    }
    char* base = static_cast<char*>(workspace);
    bool any_copy = false;
    for (size_t g = 0; g < ngroups; ++g) {
        const int32_t b0 = b[g], b1 = b[g + 1];
        const std::vector<mfsdp_owner_segments> gs = segs_without_copies(segs, b0, b1);
        st = muon_step_impl(mats + b0, gs.data(), b1 - b0, hp, base + off[g], sz[g], stream);
        if (st) {
            release();
            return st;
        }
        bool copies = false;
        for (int32_t i = b0; i < b1; ++i) copies = copies || (segs[i].ncopies > 0 && mats[i].rows > 0 && mats[i].cols > 0);
        if (!copies) continue;
        any_copy = true;
        // this group's parameters are final once its write kernel is done: move
        // them on the copy engines while the next groups compute
        if (cudaEventRecord(ev[g], s) != cudaSuccess || cudaStreamWaitEvent(cs, ev[g], 0) != cudaSuccess) {
            cudaGetLastError();
            release();
            return MFSDP_ERR_CUDA;
        }
        for (int32_t i = b0; i < b1; ++i) {
            const mfsdp_matrix& m = mats[i];
            if (m.rows == 0 || m.cols == 0) continue;
            const size_t nbytes = static_cast<size_t>(m.rows * m.cols) * (m.param_dtype == MFSDP_DTYPE_BF16 ? 2 : 4);
            for (int32_t d = 0; d < segs[i].ncopies; ++d) {
                if (cudaMemcpyAsync(segs[i].param_copies[d], m.param, nbytes, cudaMemcpyDefault, cs) != cudaSuccess) {
                    cudaGetLastError();
                    release();
                    return MFSDP_ERR_CUDA;
                }
            }
        }
    }
    if (any_copy) {
        // the caller's stream completes only after every copy
        if (cudaEventRecord(ev[ngroups], cs) != cudaSuccess || cudaStreamWaitEvent(s, ev[ngroups], 0) != cudaSuccess) {
            cudaGetLastError();
            release();
            return MFSDP_ERR_CUDA;
        }
    }
    release();
    return MFSDP_OK;
}

int mfsdp::muon_step_impl(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n,
                          const mfsdp_muon_hparams* hp, void* workspace, size_t workspace_bytes, void* stream,
                          bool always_upload) {
    int st = validate_all(mats, segs, n, hp);
    if (st) return st;
    int32_t live = 0;
    for (int32_t i = 0; i < n; ++i) live += (mats[i].rows > 0 && mats[i].cols > 0);
    if (live == 0) return MFSDP_OK;
    st = check_device();
    if (st) return st;
    if (!workspace) return MFSDP_ERR_INVALID_ARG;
    if (!aligned(workspace, kAlign)) return MFSDP_ERR_MISALIGNED;
    int max_clusters = 1;
    if (pick_engine(hp) == Engine::Tc) {
        max_clusters = tc_max_clusters();
        if (max_clusters <= 0) return MFSDP_ERR_CUDA;
    }
    Layout L;
    char* base = static_cast<char*>(workspace);
    st = build_layout(mats, segs, n, hp, base, L, max_clusters);
    if (st) return st;
    if (workspace_bytes < L.total) return MFSDP_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // head bytes: descriptor table and tile tables
    std::vector<char> head(L.off_partials, 0);
    std::memcpy(head.data() + L.off_mats, L.mats.data(), L.mats.size() * sizeof(MatDev));
    if (!L.ptrs.empty())
        std::memcpy(head.data() + L.off_ptrs, L.ptrs.data(), L.ptrs.size() * sizeof(uint64_t));
    if (L.maps_bytes && !tc_encode_maps(L.mats, head.data() + L.off_maps)) return MFSDP_ERR_CUDA;
    if (!L.sym_tiles.empty())
        std::memcpy(head.data() + L.off_sym, L.sym_tiles.data(), L.sym_tiles.size() * sizeof(TileDev));
    if (!L.poly_tiles.empty())
        std::memcpy(head.data() + L.off_poly, L.poly_tiles.data(), L.poly_tiles.size() * sizeof(TileDev));
    if (!L.gen_tiles.empty())
        std::memcpy(head.data() + L.off_gen, L.gen_tiles.data(), L.gen_tiles.size() * sizeof(TileDev));
    auto put_seg = [&](size_t off, const std::vector<int32_t>& seg) {
        if (!seg.empty()) std::memcpy(head.data() + off, seg.data(), seg.size() * sizeof(int32_t));
    };
    put_seg(L.off_sym_seg, L.sym_seg);
    put_seg(L.off_poly_seg, L.poly_seg);
    put_seg(L.off_gen_seg, L.gen_seg);
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lock(g_cache_mu);
        auto it = g_cache.find(reinterpret_cast<uintptr_t>(workspace));
        const bool fresh = !always_upload && it != g_cache.end() && it->second.dev == dev && it->second.head == head;
        if (!fresh) {
            if (cudaMemcpyAsync(base, head.data(), head.size(), cudaMemcpyHostToDevice, s) != cudaSuccess) {
                cudaGetLastError();
                g_cache.erase(reinterpret_cast<uintptr_t>(workspace));
                return MFSDP_ERR_CUDA;
            }
            // a shared scratch (always_upload) is never assumed to still hold this head
            if (always_upload) g_cache.erase(reinterpret_cast<uintptr_t>(workspace));
            else g_cache[reinterpret_cast<uintptr_t>(workspace)] = CacheEntry{dev, std::move(head)};
        }
    }
    const MatDev* d_mats = reinterpret_cast<const MatDev*>(base + L.off_mats);
    const TileDev* d_sym = reinterpret_cast<const TileDev*>(base + L.off_sym);
    const TileDev* d_poly = reinterpret_cast<const TileDev*>(base + L.off_poly);
    const void* d_maps = base + L.off_maps;
    const TileDev* d_gen = reinterpret_cast<const TileDev*>(base + L.off_gen);
    float* d_partials = reinterpret_cast<float*>(base + L.off_partials);
    float* d_s = reinterpret_cast<float*>(base + L.off_s);
    const int32_t nm = static_cast<int32_t>(L.mats.size());

    StepScalars sc{};
    sc.a = hp->a; sc.b = hp->b; sc.c = hp->c;
    sc.lr = hp->lr;
    sc.decay = static_cast<float>(1.0 - static_cast<double>(hp->lr) * hp->weight_decay);
    sc.beta = hp->beta;
    sc.eps = hp->eps;
    sc.nesterov = hp->nesterov;
    sc.bf16_mode = hp->mode == MFSDP_MODE_BF16;

    int slot = prof_before(MFSDP_KCLASS_MOMENTUM, s);
    // the flat groups stream through bulk copies when every flat matrix has the dtypes those kernels take
    bool grads_bf16 = true, params_bf16 = true;
    for (const MatDev& m : L.mats) {
        if (!m.mom_flat) continue;
        grads_bf16 = grads_bf16 && m.grad_bf16;
        params_bf16 = params_bf16 && m.param_bf16;
    }
    cudaError_t e = launch_momentum(d_mats, nm, L.flat_groups, L.mom_groups, sc, d_partials, segs != nullptr,
                                    grads_bf16, s);
    prof_after(slot, s);
    if (e != cudaSuccess) return MFSDP_ERR_CUDA;
    slot = prof_before(MFSDP_KCLASS_NORM, s);
    e = launch_norm(d_mats, nm, d_partials, d_s, hp->eps, s);
    prof_after(slot, s);
    if (e != cudaSuccess) return MFSDP_ERR_CUDA;
    const int32_t nsym = static_cast<int32_t>(L.sym_tiles.size());
    const int32_t ngen = static_cast<int32_t>(L.gen_tiles.size());
    const int32_t* d_sym_seg = reinterpret_cast<const int32_t*>(base + L.off_sym_seg);
    const int32_t* d_poly_seg = reinterpret_cast<const int32_t*>(base + L.off_poly_seg);
    const int32_t* d_gen_seg = reinterpret_cast<const int32_t*>(base + L.off_gen_seg);
    auto clusters = [](const std::vector<int32_t>& seg) { return static_cast<int32_t>(seg.size()) - 1; };
    const bool tc = L.engine == Engine::Tc;
    const int32_t ring_gram = tc ? tc_ring_depth(PH_GRAM, L.mats, nsym, clusters(L.sym_seg)) : 0;
    const int32_t ring_poly = tc ? tc_ring_depth(PH_POLY, L.mats, nsym, clusters(L.poly_seg)) : 0;
    const int32_t ring_gen = tc ? tc_ring_depth(PH_APPLY, L.mats, ngen, clusters(L.gen_seg)) : 0;
    auto gemm = [&](Phase ph, const TileDev* tiles, int32_t ntiles, const int32_t* d_seg, int32_t nclus, int32_t it,
                    int cls) {
        const int sl = prof_before(cls, s);
        const cudaError_t r = L.engine == Engine::Tc
                                  ? launch_gemm_tc(ph, d_mats, d_maps, nm, tiles, d_seg, nclus, it,
                                                   ph == PH_GRAM ? ring_gram : ph == PH_POLY ? ring_poly : ring_gen,
                                                   sc, d_s, s)
                                  : launch_gemm_simt(ph, d_mats, nm, tiles, ntiles, it, sc, d_s, s);
        prof_after(sl, s);
        return r;
    };
    for (int32_t it = 0; it < hp->ns_steps; ++it) {
        const bool last = it == hp->ns_steps - 1;
        e = gemm(PH_GRAM, d_sym, nsym, d_sym_seg, clusters(L.sym_seg), it, MFSDP_KCLASS_GRAM);
        if (e == cudaSuccess) e = gemm(PH_POLY, d_poly, nsym, d_poly_seg, clusters(L.poly_seg), it, MFSDP_KCLASS_POLY);
        if (e == cudaSuccess)
            e = gemm(last ? PH_FINAL : PH_APPLY, d_gen, ngen, d_gen_seg, clusters(L.gen_seg), it,
                     last ? MFSDP_KCLASS_FINAL : MFSDP_KCLASS_APPLY);
        if (e != cudaSuccess) return MFSDP_ERR_CUDA;
    }
    // the parameter write reads X from the master copy the last iteration wrote
    // (iteration it reads copy it & 1 and writes the other)
    const int32_t xsel = hp->ns_steps & 1;
    slot = prof_before(MFSDP_KCLASS_WRITE, s);
    e = launch_param_write(d_mats, nm, L.flat_groups, L.mom_groups, sc, d_s, xsel, hp->ns_steps == 0 ? 1 : 0,
                           params_bf16 && sc.bf16_mode, s);
    prof_after(slot, s);
    if (e != cudaSuccess) return MFSDP_ERR_CUDA;
    return MFSDP_OK;
}

extern "C" int mfsdp_adamw_tail(float* p, const float* g, float* m, float* v, int64_t n,
                                const mfsdp_adamw_hparams* hp, void* stream) {
    if (!hp || n < 0) return MFSDP_ERR_INVALID_ARG;
    if (hp->step < 1) return MFSDP_ERR_INVALID_ARG;
    if (!std::isfinite(hp->lr) || !std::isfinite(hp->beta1) || !std::isfinite(hp->beta2) ||
        !std::isfinite(hp->eps) || !std::isfinite(hp->weight_decay))
        return MFSDP_ERR_INVALID_ARG;
    if (hp->beta1 < 0.f || hp->beta1 >= 1.f || hp->beta2 < 0.f || hp->beta2 >= 1.f)
        return MFSDP_ERR_INVALID_ARG;
    if (n == 0) return MFSDP_OK;
    if (!p || !g || !m || !v) return MFSDP_ERR_INVALID_ARG;
    if (!aligned(p, 4) || !aligned(g, 4) || !aligned(m, 4) || !aligned(v, 4)) return MFSDP_ERR_MISALIGNED;
    // the four buffers must not overlap
    {
        const uintptr_t len = static_cast<uintptr_t>(n) * 4;
        const uintptr_t b[4] = {reinterpret_cast<uintptr_t>(p), reinterpret_cast<uintptr_t>(g),
                                reinterpret_cast<uintptr_t>(m), reinterpret_cast<uintptr_t>(v)};
        for (int i = 0; i < 4; ++i)
            for (int j = i + 1; j < 4; ++j)
                if (b[i] < b[j] + len && b[j] < b[i] + len) return MFSDP_ERR_INVALID_ARG;
    }
    int st = check_device();
    if (st) return st;
    const double t = static_cast<double>(hp->step);
    const float bc1 = static_cast<float>(1.0 - std::pow(static_cast<double>(hp->beta1), t));
    const float bc2 = static_cast<float>(1.0 - std::pow(static_cast<double>(hp->beta2), t));
    const float decay = static_cast<float>(1.0 - static_cast<double>(hp->lr) * hp->weight_decay);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int slot = prof_before(MFSDP_KCLASS_ADAMW, s);
    const cudaError_t e = launch_adamw(p, g, m, v, n, hp->lr, hp->beta1, hp->beta2, hp->eps, decay, bc1, bc2, s);
    prof_after(slot, s);
    return e == cudaSuccess ? MFSDP_OK : MFSDP_ERR_CUDA;
}

extern "C" int mfsdp_selftest_bounded_wait(int64_t limit_ns, void* stream) {
    if (limit_ns < 1000 || limit_ns > 10000000000LL) return MFSDP_ERR_INVALID_ARG;
    int st = check_device();
    if (st) return st;
    return launch_bounded_wait_selftest(static_cast<unsigned long long>(limit_ns), static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? MFSDP_OK
               : MFSDP_ERR_CUDA;
}

extern "C" int mfsdp_get_device_status(void* stream, int32_t* status) {
    if (!status) return MFSDP_ERR_INVALID_ARG;
    int32_t* d = device_status_ptr();
    if (!d) return MFSDP_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t h = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) { cudaGetLastError(); return MFSDP_ERR_CUDA; }
    if (cudaMemcpy(&h, d, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) { cudaGetLastError(); return MFSDP_ERR_CUDA; }
    const int32_t zero = 0;
    if (cudaMemcpy(d, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) { cudaGetLastError(); return MFSDP_ERR_CUDA; }
    *status = h;
    return MFSDP_OK;
}

extern "C" const char* mfsdp_status_string(int32_t status) {
    switch (status) {
        case MFSDP_OK: return "MFSDP_OK";
        case MFSDP_ERR_INVALID_ARG: return "MFSDP_ERR_INVALID_ARG: invalid argument";
        case MFSDP_ERR_UNSUPPORTED_DTYPE: return "MFSDP_ERR_UNSUPPORTED_DTYPE: unsupported dtype";
        case MFSDP_ERR_MISALIGNED: return "MFSDP_ERR_MISALIGNED: misaligned pointer";
        case MFSDP_ERR_WORKSPACE_TOO_SMALL: return "MFSDP_ERR_WORKSPACE_TOO_SMALL: workspace too small";
        case MFSDP_ERR_CUDA: return "MFSDP_ERR_CUDA: CUDA runtime error";
        case MFSDP_ERR_TIMEOUT: return "MFSDP_ERR_TIMEOUT: bounded device wait gave up";
        case MFSDP_ERR_DEVICE_FAULT: return "MFSDP_ERR_DEVICE_FAULT: kernel skipped an out-of-range index";
        case MFSDP_ERR_UNSUPPORTED_DEVICE: return "MFSDP_ERR_UNSUPPORTED_DEVICE: device is not sm_100";
        default: return "unknown mfsdp status";
    }
}

extern "C" int32_t mfsdp_version(void) { return 100; }
