// Host-side balance-aware owner planner and MatrixShard records.
//
// Passage: "MatrixFSDP: communication-free matrix optimizers under ZeRO-3
// parameter sharding", arxivlens summary page, Abstract (each 2D weight owned
// whole by one data-parallel rank, empty shards elsewhere; non-matrix tensors
// packed into tail owners; MatrixShard metadata and a balance-aware owner
// planner) and the gist.science French summary, Methodologie section 2,
// "Metadonnees MatrixShard & Planificateur Global" (owners balance resident
// bytes and optimizer workload).  The pages give no algorithm; this is a
// greedy longest-processing-time assignment over two balanced resources,
// Newton-Schulz FLOPs and resident bytes.
#include "../../include/mfsdp.h"

#include <algorithm>
#include <cstdint>
#include <cmath>
#include <vector>

namespace {

struct Item {
    int64_t id;
    double f;     // Newton-Schulz FLOPs (dense count)
    int64_t b;    // resident bytes
};

double ns_cost(int64_t rows, int64_t cols, int32_t steps) {
    const int64_t r = std::min(rows, cols), c = std::max(rows, cols);
    // exact in int64 for every realistic shape (< 2^63), then one conversion
    const int64_t per = 4 * r * r * c + 2 * r * r * r;
    return static_cast<double>(per * static_cast<int64_t>(steps));
}

int64_t bytes_of(const mfsdp_param_desc& p) {
    const int64_t n = p.rows * p.cols;
    if (p.kind != MFSDP_KIND_MATRIX) return 16 * n;  // p, g, m, v in fp32
    const int64_t e = (p.dtype == MFSDP_DTYPE_BF16) ? 2 : 4;
    return n * (e + e + 4);                           // param + grad + fp32 momentum
}

}  // namespace

extern "C" int mfsdp_plan(const mfsdp_param_desc* params, int64_t n, int32_t world_size, int32_t ns_steps,
                          mfsdp_matrix_shard* out, double* out_rank_flops, int64_t* out_rank_bytes) {
    if (n < 0 || world_size < 1 || ns_steps < 0) return MFSDP_ERR_INVALID_ARG;
    if (n > 0 && (!params || !out)) return MFSDP_ERR_INVALID_ARG;
    for (int64_t i = 0; i < n; ++i) {
        const mfsdp_param_desc& p = params[i];
        if (p.rows < 0 || p.cols < 0) return MFSDP_ERR_INVALID_ARG;
        if (p.kind != MFSDP_KIND_MATRIX && p.kind != MFSDP_KIND_TAIL) return MFSDP_ERR_INVALID_ARG;
        if (p.kind == MFSDP_KIND_MATRIX && p.dtype != MFSDP_DTYPE_F32 && p.dtype != MFSDP_DTYPE_BF16)
            return MFSDP_ERR_UNSUPPORTED_DTYPE;
    }
    const int R = world_size;
    std::vector<Item> mats;
    double total_f = 0.0;
    int64_t total_b = 0;
    int64_t tail_bytes = 0;
    bool has_tail = false;
    for (int64_t i = 0; i < n; ++i) {
        if (params[i].kind == MFSDP_KIND_MATRIX) {
            Item it{i, ns_cost(params[i].rows, params[i].cols, ns_steps), bytes_of(params[i])};
            total_f += it.f;
            total_b += it.b;
            mats.push_back(it);
        } else {
            has_tail = true;
            tail_bytes += bytes_of(params[i]);
        }
    }
    std::sort(mats.begin(), mats.end(), [](const Item& x, const Item& y) {
        if (x.f != y.f) return x.f > y.f;
        if (x.b != y.b) return x.b > y.b;
        return x.id < y.id;
    });
    const double fbar = total_f / R;
    const double bbar = static_cast<double>(total_b) / R;
    std::vector<double> F(R, 0.0);
    std::vector<int64_t> B(R, 0);
    std::vector<int32_t> owner(static_cast<size_t>(n), 0);
    for (const Item& it : mats) {
        int best = -1;
        double best_score = 0.0, best_load = 0.0;
        for (int r = 0; r < R; ++r) {
            const double load = F[r] + it.f;
            const double rf = fbar > 0.0 ? load / fbar : 0.0;
            const double rb = bbar > 0.0 ? static_cast<double>(B[r] + it.b) / bbar : 0.0;
            const double score = rf > rb ? rf : rb;
            // lexicographic (score, load, rank): a later rank wins only when strictly better
            if (best < 0 || score < best_score || (score == best_score && load < best_load)) {
                best = r;
                best_score = score;
                best_load = load;
            }
        }
        owner[static_cast<size_t>(it.id)] = best;
        F[best] += it.f;
        B[best] += it.b;
    }
    if (has_tail) {
        int t = 0;
        for (int r = 1; r < R; ++r)
            if (B[r] < B[t]) t = r;
        for (int64_t i = 0; i < n; ++i)
            if (params[i].kind != MFSDP_KIND_MATRIX) owner[static_cast<size_t>(i)] = t;
        B[t] += tail_bytes;
    }
    // owner-local offsets: parameter-id order within each owner; tails in one packed buffer
    std::vector<int64_t> next(R, 0);
    int64_t tail_off = 0;
    for (int64_t i = 0; i < n; ++i) {
        const mfsdp_param_desc& p = params[i];
        mfsdp_matrix_shard& s = out[i];
        const bool is_mat = p.kind == MFSDP_KIND_MATRIX;
        s.param_id = i;
        s.rows = p.rows;
        s.cols = p.cols;
        s.owner = owner[static_cast<size_t>(i)];
        s.kind = is_mat ? MFSDP_KIND_MATRIX : MFSDP_KIND_TAIL;
        s.transposed = (is_mat && p.rows > p.cols) ? 1 : 0;
        s.reserved = 0;
        s.ns_flops = is_mat ? ns_cost(p.rows, p.cols, ns_steps) : 0.0;
        s.resident_bytes = bytes_of(p);
        if (is_mat) {
            s.owner_offset = next[s.owner];
            next[s.owner] += p.rows * p.cols;
            s.shape_scale = (p.cols > 0 && p.rows > p.cols)
                                ? std::sqrt(static_cast<double>(p.rows) / static_cast<double>(p.cols))
                                : 1.0;
        } else {
            s.owner_offset = tail_off;
            tail_off += p.rows * p.cols;
            s.shape_scale = 1.0;
        }
    }
    if (out_rank_flops)
        for (int r = 0; r < R; ++r) out_rank_flops[r] = F[r];
    if (out_rank_bytes)
        for (int r = 0; r < R; ++r) out_rank_bytes[r] = B[r];
    return MFSDP_OK;
}

extern "C" int mfsdp_heaviest_rank(const double* rank_flops, const int64_t* rank_bytes, int32_t world_size,
                                   int32_t* out_rank) {
    if (!rank_flops || !rank_bytes || !out_rank || world_size < 1) return MFSDP_ERR_INVALID_ARG;
    int h = 0;
    for (int r = 1; r < world_size; ++r) {
        if (rank_flops[r] > rank_flops[h] ||
            (rank_flops[r] == rank_flops[h] && rank_bytes[r] > rank_bytes[h]))
            h = r;
    }
    *out_rank = h;
    return MFSDP_OK;
}

// Owner-shard checkpoint resharding.  Passage: gist.science French summary,
// Methodologie section 2, "Checkpointing et Routage" (saved placement layout,
// optimizer state routed to its owners through the MatrixShard metadata,
// restore across world sizes).  The new layout is the planner's own answer for
// the new world size; each parameter's state goes from its saved (owner,
// offset) to its new one.
extern "C" int mfsdp_reshard(const mfsdp_param_desc* params, const mfsdp_matrix_shard* saved, int64_t n,
                             int32_t new_world_size, int32_t ns_steps, mfsdp_matrix_shard* out_shards,
                             mfsdp_reshard_route* out_routes, int64_t* out_moved_bytes) {
    if (n < 0 || new_world_size < 1) return MFSDP_ERR_INVALID_ARG;
    if (n > 0 && (!params || !saved || !out_shards || !out_routes)) return MFSDP_ERR_INVALID_ARG;
    for (int64_t i = 0; i < n; ++i) {
        const mfsdp_param_desc& p = params[i];
        const mfsdp_matrix_shard& s = saved[i];
        const int32_t kind = p.kind == MFSDP_KIND_MATRIX ? MFSDP_KIND_MATRIX : MFSDP_KIND_TAIL;
        if (s.param_id != i || s.rows != p.rows || s.cols != p.cols || s.kind != kind) return MFSDP_ERR_INVALID_ARG;
        if (s.owner < 0 || s.owner_offset < 0) return MFSDP_ERR_INVALID_ARG;
    }
    const int st = mfsdp_plan(params, n, new_world_size, ns_steps, out_shards, nullptr, nullptr);
    if (st != MFSDP_OK) return st;
    int64_t moved = 0;
    for (int64_t i = 0; i < n; ++i) {
        const mfsdp_param_desc& p = params[i];
        const bool is_mat = p.kind == MFSDP_KIND_MATRIX;
        const int64_t elems = p.rows * p.cols;
        mfsdp_reshard_route& r = out_routes[i];
        r.param_id = i;
        r.kind = is_mat ? MFSDP_KIND_MATRIX : MFSDP_KIND_TAIL;
        r.src_rank = saved[i].owner;
        r.dst_rank = out_shards[i].owner;
        r.reserved = 0;
        r.src_offset = saved[i].owner_offset;
        r.dst_offset = out_shards[i].owner_offset;
        r.elems = elems;
        r.state_bytes = is_mat ? elems * ((p.dtype == MFSDP_DTYPE_BF16 ? 2 : 4) + 4) : elems * 12;
        if (r.src_rank != r.dst_rank) moved += r.state_bytes;
    }
    if (out_moved_bytes) *out_moved_bytes = moved;
    return MFSDP_OK;
}
