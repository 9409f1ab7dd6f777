// Structure-aware bucket planner (host C++, runs once at init).
//
// veScale-FSDP (paper Sec. 4, page section "2. Structure-aware planning
// algorithm"): tensors of a bucket are ordered by block size, largest first,
// then placed by a dynamic program over offsets so that every boundary
// between the m per-device slices falls on a block edge of the tensor it cuts
// (RaggedShard blocks are never split) and padding sits only between
// tensors.  The pages quote O(|T|^2 m log E log(|T| m)) for their DP; this
// planner is exact for the same objective and faster:
//
//  * For a fixed order and slice size s the DP's state collapses to the end
//    of the last placed tensor: a tensor's set of allowed starts does not
//    depend on earlier tensors, and an earlier end never removes a later
//    option, so the earliest allowed start is optimal for every tensor.
//  * The earliest allowed start is found in O(1): either the tensor fits in
//    the rest of the current slice, or it must cross the next boundary R on a
//    block edge, i.e. start at R - j with j a positive multiple of
//    lcm(align, b); the smallest such start is the only candidate in this
//    slice.  Failing that, the next slice start is tried once; every later
//    slice start repeats its outcome (same relative position) except that the
//    bucket end comes closer.
//  * Feasibility is not monotone in s, so s is scanned upward from the even
//    share; a tensor longer than 2s always holds two consecutive boundaries,
//    which forces its block size to divide s.  Within a range of s where the
//    set of such tensors is fixed, only multiples of the lcm of their block
//    sizes (and align) are tried.
#include <algorithm>
#include <cstring>
#include <limits>
#include <new>
#include <numeric>

#include "internal.h"

namespace {

constexpr int64_t kInf = std::numeric_limits<int64_t>::max() / 4;

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t up(int64_t a, int64_t q) { return cdiv(a, q) * q; }

// lcm with saturation at kInf.
int64_t lcm_sat(int64_t a, int64_t b) {
    if (a >= kInf || b >= kInf) return kInf;
    int64_t g = std::gcd(a, b);
    int64_t r;
    if (__builtin_mul_overflow(a / g, b, &r) || r >= kInf) return kInf;
    return r;
}

struct Item {
    int64_t n, b, lcm_ab;
    int32_t id;
};

// Earliest start >= lo for one tensor at slice size s, or -1.
int64_t earliest(const Item& t, int64_t lo, int64_t s, int64_t m, int64_t A) {
    const int64_t end = m * s;
    int64_t o = up(lo, A);
    for (int attempt = 0; attempt < 2; ++attempt) {
        if (o + t.n > end) return -1;
        const int64_t R = (o / s + 1) * s;
        if (o + t.n <= R) return o;
        const int64_t j = t.lcm_ab >= kInf ? 0 : ((R - o) / t.lcm_ab) * t.lcm_ab;
        if (j > 0) {
            const int64_t c = R - j;
            if (c + t.n > end) return -1;
            if (c + t.n <= R + s || s % t.b == 0) return c;
        }
        o = R;  // only the next slice start is left to try (see header)
    }
    return -1;
}

bool place(const std::vector<Item>& items, int64_t s, int64_t m, int64_t A, std::vector<int64_t>& off) {
    int64_t lo = 0;
    for (const Item& t : items) {
        int64_t o = earliest(t, lo, s, m, A);
        if (o < 0) return false;
        off[t.id] = o;
        lo = o + t.n;
    }
    return true;
}

}  // namespace

extern "C" dbuf_status dbuf_plan(const dbuf_tensor_desc* descs, int32_t n, int32_t m,
                                 int64_t align_elems, int64_t max_bucket_elems, dbuf_plan_t** out) {
    using dbuf_detail::fail;
    if (!out) return fail(DBUF_EINVAL, "dbuf_plan: out is NULL");
    *out = nullptr;
    if (n < 0 || (n > 0 && !descs)) return fail(DBUF_EINVAL, "dbuf_plan: bad tensor list");
    if (m < 1) return fail(DBUF_EINVAL, "dbuf_plan: m must be >= 1");
    if (align_elems < 1 || align_elems > (int64_t(1) << 30))
        return fail(DBUF_EINVAL, "dbuf_plan: align_elems must be in [1, 2^30]");
    if (max_bucket_elems < 0) return fail(DBUF_EINVAL, "dbuf_plan: max_bucket_elems < 0");
    const int64_t A = align_elems;

    std::vector<Item> items(n);
    int64_t total = 0, upper = 0;
    for (int32_t i = 0; i < n; ++i) {
        const dbuf_tensor_desc& d = descs[i];
        if (d.rows < 1 || d.cols < 1 || d.k < 1 || d.k > d.rows || d.block_cols < 0)
            return fail(DBUF_EINVAL, "dbuf_plan: tensor " + std::to_string(i) +
                                         " needs rows, cols, k >= 1, k <= rows and block_cols >= 0");
        if (d.block_cols > 0 && d.block_cols < d.cols &&
            (d.block_cols < 16 || d.block_cols > 4096 || (d.block_cols & (d.block_cols - 1)) != 0 || d.cols % 16 != 0))
            return fail(DBUF_EINVAL, "dbuf_plan: tensor " + std::to_string(i) +
                                         " tiles need block_cols a power of two in [16, 4096] and cols % 16 == 0");
        if (d.block_cols > 0 && d.block_cols < d.cols && (d.k > (int64_t(1) << 30) || d.cols > (int64_t(1) << 30)))
            return fail(DBUF_EINVAL, "dbuf_plan: tensor " + std::to_string(i) + " tiles need k, cols <= 2^30");
        int64_t ne, be;
        if (__builtin_mul_overflow(d.rows, d.cols, &ne) || ne > (int64_t(1) << 46))
            return fail(DBUF_EINVAL, "dbuf_plan: tensor " + std::to_string(i) + " too large");
        be = d.k * d.cols;
        items[i] = Item{ne, be, lcm_sat(A, be), i};
        total += ne;
        upper += up(ne, A);
    }
    upper = up(upper, A);  // every tensor in slice 0: always placeable
    std::sort(items.begin(), items.end(), [](const Item& x, const Item& y) {
        if (x.b != y.b) return x.b > y.b;
        if (x.n != y.n) return x.n > y.n;
        return x.id < y.id;
    });

    std::vector<int64_t> off(n, 0);
    int64_t s = up(cdiv(total, m), A);
    bool found = (total == 0);
    if (!found) {
        // Tensors by element count, descending: the ones longer than 2s form a
        // prefix of this list that shrinks as s grows.
        std::vector<int32_t> by_n(n);
        std::iota(by_n.begin(), by_n.end(), 0);
        std::vector<Item> byid(n);
        for (const Item& t : items) byid[t.id] = t;
        std::sort(by_n.begin(), by_n.end(), [&](int32_t a, int32_t b) { return byid[a].n > byid[b].n; });
        while (s <= upper) {
            int32_t big = 0;
            while (big < n && byid[by_n[big]].n > 2 * s) ++big;
            int64_t L = A;
            for (int32_t i = 0; i < big && L < kInf; ++i) L = lcm_sat(L, byid[by_n[i]].b);
            // Next s at which the prefix shrinks: the shortest long tensor
            // stops being longer than 2s at s = ceil(n/2).
            const int64_t next_regime = big > 0 ? cdiv(byid[by_n[big - 1]].n, 2) : kInf;
            const int64_t c = L >= kInf ? kInf : up(s, L);
            if (c >= next_regime) {
                s = up(next_regime, A);
                continue;
            }
            if (c > upper) break;
            if (max_bucket_elems > 0 && c * m > max_bucket_elems) break;
            if (place(items, c, m, A, off)) {
                s = c;
                found = true;
                break;
            }
            s = c + A;
        }
    }
    if (!found) {
        if (max_bucket_elems > 0)
            return fail(DBUF_EINFEASIBLE, "dbuf_plan: no layout fits in max_bucket_elems");
        return fail(DBUF_EINFEASIBLE, "dbuf_plan: no layout found");  // not expected
    }
    if (max_bucket_elems > 0 && s * m > max_bucket_elems)
        return fail(DBUF_EINFEASIBLE, "dbuf_plan: no layout fits in max_bucket_elems");

    dbuf_plan_s* p = new (std::nothrow) dbuf_plan_s;
    if (!p) return fail(DBUF_ENOMEM, "dbuf_plan: out of host memory");
    p->n = n;
    p->m = m;
    p->align = A;
    p->slice = total == 0 ? 0 : s;
    p->bucket = p->slice * m;
    p->padding = p->bucket - total;
    p->rows.resize(n);
    p->cols.resize(n);
    p->k.resize(n);
    p->tile_cols.resize(n);
    p->offset = off;
    int64_t nb = 0;
    for (int32_t i = 0; i < n; ++i) {
        p->rows[i] = descs[i].rows;
        p->cols[i] = descs[i].cols;
        p->k[i] = descs[i].k;
        const int64_t bc = descs[i].block_cols;
        p->tile_cols[i] = (bc > 0 && bc < descs[i].cols) ? bc : 0;
        const int64_t per_row_block = p->tile_cols[i] ? cdiv(descs[i].cols, p->tile_cols[i]) : 1;
        nb += cdiv(descs[i].rows, descs[i].k) * per_row_block;
    }
    p->n_blocks = nb;
    p->by_offset.resize(n);
    std::iota(p->by_offset.begin(), p->by_offset.end(), 0);
    std::stable_sort(p->by_offset.begin(), p->by_offset.end(),
                     [&](int32_t a, int32_t b) { return off[a] < off[b]; });
    *out = p;
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_plan_info(const dbuf_plan_t* plan, int64_t* slice_elems,
                                      int64_t* bucket_elems, int64_t* padding_elems, int64_t* n_blocks,
                                      int64_t* offsets) {
    if (!plan) return dbuf_detail::fail(DBUF_EINVAL, "dbuf_plan_info: plan is NULL");
    if (slice_elems) *slice_elems = plan->slice;
    if (bucket_elems) *bucket_elems = plan->bucket;
    if (padding_elems) *padding_elems = plan->padding;
    if (n_blocks) *n_blocks = plan->n_blocks;
    if (offsets && plan->n) std::memcpy(offsets, plan->offset.data(), sizeof(int64_t) * plan->n);
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_plan_dims(const dbuf_plan_t* plan, int32_t* n_tensors, int32_t* m) {
    if (!plan) return dbuf_detail::fail(DBUF_EINVAL, "dbuf_plan_dims: plan is NULL");
    if (n_tensors) *n_tensors = plan->n;
    if (m) *m = plan->m;
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_plan_shards(const dbuf_plan_t* plan, dbuf_shard_rows* out) {
    if (!plan) return dbuf_detail::fail(DBUF_EINVAL, "dbuf_plan_shards: plan is NULL");
    if (plan->n > 0 && !out) return dbuf_detail::fail(DBUF_EINVAL, "dbuf_plan_shards: out is NULL");
    const int64_t s = plan->slice;
    for (int32_t i = 0; i < plan->n; ++i) {
        const int64_t o = plan->offset[i], c = plan->cols[i], n = plan->rows[i] * c;
        for (int32_t r = 0; r < plan->m; ++r) {
            // The part of the tensor inside slice r, in elements from its start;
            // interior slice boundaries are block edges, so whole rows.
            const int64_t a = std::min(n, std::max<int64_t>(0, (int64_t)r * s - o));
            const int64_t b = std::min(n, std::max<int64_t>(0, (int64_t)(r + 1) * s - o));
            out[(int64_t)i * plan->m + r] = dbuf_shard_rows{a / c, std::max(a, b) / c};
        }
    }
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_plan_rank(const dbuf_plan_t* plan, int32_t rank, dbuf_plan_t** out,
                                      int64_t* first_block) {
    using dbuf_detail::fail;
    if (!out) return fail(DBUF_EINVAL, "dbuf_plan_rank: out is NULL");
    *out = nullptr;
    if (!plan) return fail(DBUF_EINVAL, "dbuf_plan_rank: plan is NULL");
    if (rank < 0 || rank >= plan->m) return fail(DBUF_EINVAL, "dbuf_plan_rank: rank must be in [0, m)");
    dbuf_plan_s* p = new (std::nothrow) dbuf_plan_s;
    if (!p) return fail(DBUF_ENOMEM, "dbuf_plan_rank: out of host memory");
    const int64_t s = plan->slice, lo = (int64_t)rank * s, hi = lo + s;
    int64_t used = 0, nb = 0, before = 0;
    for (int32_t i = 0; i < plan->n; ++i) {
        const int64_t o = plan->offset[i], c = plan->cols[i], K = plan->k[i], n = plan->rows[i] * c;
        const int64_t tc = plan->tile_cols.empty() ? 0 : plan->tile_cols[i];
        const int64_t G = tc ? cdiv(c, tc) : 1;  // blocks per k-row block
        // Elements [a, b) of the tensor lie in the slice.  Interior slice
        // boundaries are k-row block edges, so both are whole rows and a is a
        // multiple of k rows.
        const int64_t a = std::min(n, std::max<int64_t>(0, lo - o));
        const int64_t b = std::max(a, std::min(n, std::max<int64_t>(0, hi - o)));
        if (a % c != 0 || b % c != 0 || (a < n && (a / c) % K != 0)) {
            delete p;
            return fail(DBUF_EINVAL, "dbuf_plan_rank: tensor " + std::to_string(i) +
                                         " is cut off a block edge (not a plan from dbuf_plan)");
        }
        before += G * cdiv(a / c, K);
        if (b == a) continue;
        p->rows.push_back((b - a) / c);
        p->cols.push_back(c);
        p->k.push_back(K);
        p->tile_cols.push_back(tc);
        p->offset.push_back(o + a - lo);
        used += b - a;
        nb += G * cdiv((b - a) / c, K);
    }
    p->n = (int32_t)p->rows.size();
    p->m = 1;
    p->align = plan->align;
    p->slice = s;
    p->bucket = s;
    p->padding = s - used;
    p->n_blocks = nb;
    p->by_offset.resize(p->n);
    std::iota(p->by_offset.begin(), p->by_offset.end(), 0);
    std::stable_sort(p->by_offset.begin(), p->by_offset.end(),
                     [&](int32_t x, int32_t y) { return p->offset[x] < p->offset[y]; });
    if (first_block) *first_block = before;
    *out = p;
    return DBUF_OK;
}

extern "C" void dbuf_plan_free(dbuf_plan_t* plan) { delete plan; }
