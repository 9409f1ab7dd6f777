// Device runtime of the ragged-bucket optimizer step (sm_100a): the C-ABI
// of include/dbuf.h apart from the planner (planner.cpp).
//
// DBuffer (veScale-FSDP paper Sec. 5, page section "3. DBuffer"): one batch
// allocation holds every bucket array of a plan; tensors are zero-copy views;
// group operations run as one launch over the whole bucket.  The kernels are
// in step_kernel.cuh (the fused 8-bit Adam step) and pack_kernel.cuh (the
// copy-in baseline); this file builds their work tables once per bucket and
// launches them on the caller's stream.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "group_kernels.cuh"
#include "internal.h"
#include "pack_kernel.cuh"
#include "step_kernel.cuh"
#include "tables.h"

// ------------------------------------------------------------------ errors

namespace dbuf_detail {
static thread_local std::string g_err;
void set_error(const std::string& msg) { g_err = msg; }
dbuf_status fail(dbuf_status st, const std::string& msg) {
    g_err = msg;
    return st;
}
}  // namespace dbuf_detail

using dbuf_detail::fail;

extern "C" const char* dbuf_last_error(void) { return dbuf_detail::g_err.c_str(); }

// ------------------------------------------------------------ work tables

namespace {

using namespace dbuf_k;

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Entries in bucket order with the element range each one reads and writes
// (a STRIP: its whole k-row block), for the chunked host-buffer step.
struct PosTiles {
    std::vector<Tile> tiles;
    std::vector<int64_t> lo, hi;
    void add(const Tile& t, int64_t a, int64_t b) {
        tiles.push_back(t);
        lo.push_back(a);
        hi.push_back(b);
    }
};

// Padding [a, b) in entries of at most kZeroChunk elements, none crossing a
// slice boundary (multiples of s; s = 0 means one slice).
void add_zero_tiles(std::vector<Tile>& out, PosTiles* pos, int64_t a, int64_t b, int64_t s) {
    for (int64_t e = a; e < b;) {
        int64_t end = std::min(b, e + kZeroChunk);
        if (s > 0) end = std::min(end, (e / s + 1) * s);
        const Tile t{e, 0, end - e, 0, TILE_ZERO, 0, 0u};
        out.push_back(t);
        if (pos) pos->add(t, t.e0, t.e0 + t.n);
        e = end;
    }
}

// Elements a LARGE or STRIP entry streams per pass (its sort key).
int64_t entry_work(const Tile& t) { return t.kind == TILE_STRIP ? t.n * (int64_t)t.nblk : t.n; }

void build_tiles(const dbuf_plan_s& p, std::vector<Tile>& tiles, PosTiles* pos = nullptr) {
    std::vector<Tile> large, whole, zero;
    int64_t blk = 0, prev_end = 0;
    for (int32_t id : p.by_offset) {
        const int64_t o = p.offset[id], n = p.rows[id] * p.cols[id], b = p.k[id] * p.cols[id];
        const int64_t nb = cdiv(p.rows[id], p.k[id]);
        if (o > prev_end) add_zero_tiles(zero, pos, prev_end, o, p.slice);
        if (!p.tile_cols.empty() && p.tile_cols[id] > 0) {
            // 2-D blocks: each k-row block in strips of at most kTile columns.
            const int64_t C = p.cols[id], W = p.tile_cols[id], G = cdiv(C, W);
            for (int64_t j = 0; j < nb; ++j) {
                const int64_t r0 = j * p.k[id], nr = std::min(p.k[id], p.rows[id] - r0);
                for (int64_t c0 = 0; c0 < C; c0 += kTile) {
                    large.push_back(Tile{o + r0 * C + c0, blk + j * G + c0 / W, std::min<int64_t>(kTile, C - c0),
                                         (int32_t)C, TILE_STRIP, (int32_t)nr, (uint32_t)W});
                    if (pos) pos->add(large.back(), o + r0 * C, o + (r0 + nr) * C);
                }
            }
            blk += nb * G;
            prev_end = o + n;
            continue;
        }
        int64_t j = 0;
        while (j < nb) {
            const int64_t e0 = o + j * b;
            if (b <= kTile) {
                const int64_t cap = kTile - (e0 & (kAlign - 1));
                // Every entry stays inside one rank's slice: blocks end on the
                // slice boundary, so the blocks before it are whole.
                const int64_t to_edge = p.slice > 0 ? ((e0 / p.slice + 1) * p.slice - e0) / b : nb - j;
                const int64_t q = std::min<int64_t>({kMaxBlk, cap / b, nb - j, std::max<int64_t>(1, to_edge)});
                if (q >= 1) {
                    const uint32_t magic = b >= 2 ? (uint32_t)(((uint64_t(1) << 32) + (uint64_t)b - 1) / (uint64_t)b) : 0u;
                    whole.push_back(Tile{e0, blk + j, std::min(q * b, n - j * b), (int32_t)b, TILE_WHOLE,
                                         (int32_t)q, magic});
                    if (pos) pos->add(whole.back(), e0, e0 + whole.back().n);
                    j += q;
                    continue;
                }
            }
            large.push_back(Tile{e0, blk + j, std::min(b, n - j * b), 0, TILE_LARGE, 1, 0u});
            if (pos) pos->add(large.back(), e0, e0 + large.back().n);
            j += 1;
        }
        blk += nb;
        prev_end = o + n;
    }
    if (prev_end < p.bucket) add_zero_tiles(zero, pos, prev_end, p.bucket, p.slice);
    // Longest work first so the tail of the grid is short tiles.
    std::stable_sort(large.begin(), large.end(),
                     [](const Tile& x, const Tile& y) { return entry_work(x) > entry_work(y); });
    tiles.clear();
    tiles.reserve(large.size() + whole.size() + zero.size());
    tiles.insert(tiles.end(), large.begin(), large.end());
    tiles.insert(tiles.end(), whole.begin(), whole.end());
    tiles.insert(tiles.end(), zero.begin(), zero.end());
}

void build_pack_chunks(const dbuf_plan_s& p, std::vector<PackChunk>& chunks, std::vector<int64_t>& first) {
    chunks.clear();
    first.assign(p.n + 1, 0);
    for (int32_t i = 0; i < p.n; ++i) {
        first[i] = (int64_t)chunks.size();
        const int64_t n = p.rows[i] * p.cols[i];
        for (int64_t e = 0; e < n; e += kPackChunk)
            chunks.push_back(PackChunk{e, p.offset[i] + e, i, (int32_t)std::min(kPackChunk, n - e)});
    }
    first[p.n] = (int64_t)chunks.size();
}

// Consecutive runs of the bucket-order entries, each covering a contiguous
// element range [lo, hi) of about `target` elements; the ranges partition
// the bucket.  A run never ends inside a k-row block's strips.
struct HostChunk {
    int64_t t0, t1, lo, hi;
};

void build_host_chunks(const PosTiles& pos, int64_t target, std::vector<HostChunk>& out) {
    out.clear();
    const int64_t n = (int64_t)pos.tiles.size();
    int64_t t0 = 0;
    while (t0 < n) {
        int64_t t1 = t0, hi = pos.hi[t0];
        while (t1 < n && (pos.lo[t1] < hi || hi - pos.lo[t0] < target)) {
            hi = std::max(hi, pos.hi[t1]);
            ++t1;
        }
        out.push_back(HostChunk{t0, t1, pos.lo[t0], hi});
        t0 = t1;
    }
}

struct Layout {
    size_t master, param, grad, mq, vq, scales, tiles, pos_tiles, chunks, status, scratch, total;
};

Layout layout_of(const dbuf_plan_s& p, size_t n_tiles, size_t n_chunks) {
    Layout L{};
    const size_t S = (size_t)p.bucket;
    size_t at = 0;
    L.master = at; at = align256(at + S * 4);
    L.param = at;  at = align256(at + S * 2);
    L.grad = at;   at = align256(at + S * 2);
    L.mq = at;     at = align256(at + S);
    L.vq = at;     at = align256(at + S);
    L.scales = at; at = align256(at + ((size_t)p.n_blocks + 2) * 8);
    L.tiles = at;  at = align256(at + n_tiles * sizeof(Tile));
    L.pos_tiles = at; at = align256(at + n_tiles * sizeof(Tile));
    L.chunks = at; at = align256(at + n_chunks * sizeof(PackChunk));
    L.status = at; at = align256(at + 16);
    L.scratch = at; at = align256(at + sizeof(NormScratch));
    L.total = at;
    return L;
}

}  // namespace

struct dbuf_s {
    dbuf_plan_s plan;
    int device = -1;
    char* base = nullptr;
    size_t bytes = 0;
    bool owns = false;
    Layout lay{};
    float* master = nullptr;
    uint16_t* param = nullptr;
    uint16_t* grad = nullptr;
    int8_t* mq = nullptr;
    uint8_t* vq = nullptr;
    float2* scales = nullptr;
    Tile* tiles = nullptr;
    Tile* pos_tiles = nullptr;   // the same entries in bucket order (host-buffer step)
    PackChunk* chunks = nullptr;
    int32_t* status = nullptr;
    NormScratch* scratch = nullptr;
    std::vector<Tile> h_tiles;
    PosTiles h_pos;
    std::vector<HostChunk> h_host_chunks;
    // Pipeline of the host-buffer step: copies in and out on their own
    // streams, overlapping the step of other chunks.
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev_start = nullptr, ev_done = nullptr;
    std::vector<cudaEvent_t> ev_in, ev_step;
    std::vector<PackChunk> h_chunks;
    std::vector<int64_t> h_chunk_first;
    int step_grid = 0;  // persistent CTAs of the step kernel
    int norm_grid = 1;  // CTAs of the norm reduction
};

static void release_pipeline(dbuf_s* db) {
    for (cudaEvent_t e : db->ev_in) if (e) cudaEventDestroy(e);
    for (cudaEvent_t e : db->ev_step) if (e) cudaEventDestroy(e);
    if (db->ev_start) cudaEventDestroy(db->ev_start);
    if (db->ev_done) cudaEventDestroy(db->ev_done);
    if (db->s_in) cudaStreamDestroy(db->s_in);
    if (db->s_out) cudaStreamDestroy(db->s_out);
}

namespace dbuf_detail {
int32_t tensors_of(const dbuf_t* db) { return db ? db->plan.n : 0; }
int device_of(const dbuf_t* db) { return db ? db->device : -1; }
}  // namespace dbuf_detail

// ----------------------------------------------------------- launches

namespace {

using namespace dbuf_k;

// The step's scalars (double, rounded to float once), each duplicated into
// a pair for the paired fp32 instructions.
StepC2 make_step_constants(const dbuf_adam_hparams& hp, float grad_scale) {
    const double B1 = hp.beta1, B2 = hp.beta2, lr = hp.lr, wd = hp.weight_decay, eps = hp.eps;
    const double t = (double)hp.step;
    const double bc1 = 1.0 - std::pow(B1, t);
    const double sq2 = std::sqrt(1.0 - std::pow(B2, t));
    auto pair = [](double x) { return make_float2((float)x, (float)x); };
    StepC2 c;
    c.b1 = pair(B1);
    c.omb1 = pair(1.0 - B1);
    c.b2 = pair(B2);
    c.omb2 = pair(1.0 - B2);
    c.eps_hat = pair(eps * sq2);
    c.step_hat = pair(lr * sq2 / bc1);
    c.decay = pair(1.0 - lr * wd);
    c.gscale = make_float2(grad_scale, grad_scale);
    return c;
}

dbuf_status check_device(const dbuf_t* db, const char* who) {
    int dev = -1;
    CUDA_TRY(cudaGetDevice(&dev), who);
    if (dev != db->device)
        return fail(DBUF_EINVAL, std::string(who) + ": current device " + std::to_string(dev) +
                                     " is not the dbuf's device " + std::to_string(db->device));
    return DBUF_OK;
}

// Persistent grid of the step kernel on the current device: as many CTAs as
// fit at once (three per SM with its shared-memory ring), never more than tiles.
dbuf_status step_grid_for(int device, size_t n_tiles, int* grid) {
    static bool attr_set[64] = {false};
    if (device >= 0 && device < 64 && !attr_set[device]) {
        CUDA_TRY(cudaFuncSetAttribute(adam8_step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStepSmem),
                 "dbuf_create: step kernel shared memory");
        attr_set[device] = true;
    }
    int sms = 0, per_sm = 0;
    CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device), "dbuf_create: SM count");
    CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, adam8_step_kernel, kStepThreads, kStepSmem),
             "dbuf_create: step kernel occupancy");
    if (per_sm < 1) return fail(DBUF_ECUDA, "dbuf_create: the step kernel does not fit on this device");
    *grid = (int)std::min<size_t>(n_tiles, (size_t)sms * (size_t)per_sm);
    return DBUF_OK;
}

}  // namespace

// ------------------------------------------------------------------- C-ABI

extern "C" size_t dbuf_required_bytes(const dbuf_plan_t* plan) {
    if (!plan) return 0;
    std::vector<Tile> tiles;
    build_tiles(*plan, tiles);
    std::vector<PackChunk> chunks;
    std::vector<int64_t> first;
    build_pack_chunks(*plan, chunks, first);
    return layout_of(*plan, tiles.size(), chunks.size()).total;
}

extern "C" dbuf_status dbuf_work_table(const dbuf_plan_t* plan, dbuf_work_item* out, int64_t cap, int64_t* n) {
    if (!plan || !n) return fail(DBUF_EINVAL, "dbuf_work_table: NULL argument");
    if (cap > 0 && !out) return fail(DBUF_EINVAL, "dbuf_work_table: out is NULL");
    std::vector<Tile> tiles;
    build_tiles(*plan, tiles);
    *n = (int64_t)tiles.size();
    static_assert(sizeof(dbuf_work_item) == sizeof(Tile), "work item mirrors the device tile");
    const int64_t m = std::min<int64_t>(cap, *n);
    for (int64_t i = 0; i < m; ++i)
        out[i] = dbuf_work_item{tiles[i].e0, tiles[i].blk0, tiles[i].n, tiles[i].b, tiles[i].kind, tiles[i].nblk,
                                tiles[i].kind == TILE_STRIP ? (int32_t)tiles[i].magic : 0};
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_create(const dbuf_plan_t* plan, void* device_base, size_t base_bytes, void* stream,
                                   dbuf_t** out) {
    if (!out) return fail(DBUF_EINVAL, "dbuf_create: out is NULL");
    *out = nullptr;
    if (!plan) return fail(DBUF_EINVAL, "dbuf_create: plan is NULL");
    if (plan->align % kAlign != 0)
        return fail(DBUF_EINVAL, "dbuf_create: plan alignment must be a multiple of 16 elements");
    dbuf_s* db = new (std::nothrow) dbuf_s;
    if (!db) return fail(DBUF_ENOMEM, "dbuf_create: out of host memory");
    db->plan = *plan;
    build_tiles(db->plan, db->h_tiles, &db->h_pos);
    // Chunks of the host-buffer pipeline: at most 16, at least 4M elements each.
    build_host_chunks(db->h_pos, std::max<int64_t>(int64_t(1) << 22, cdiv(db->plan.bucket, 16)),
                      db->h_host_chunks);
    build_pack_chunks(db->plan, db->h_chunks, db->h_chunk_first);
    db->lay = layout_of(db->plan, db->h_tiles.size(), db->h_chunks.size());
    db->bytes = db->lay.total;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaGetDevice(&db->device);
    if (e != cudaSuccess) {
        delete db;
        return fail(DBUF_ECUDA, std::string("dbuf_create: cudaGetDevice: ") + cudaGetErrorString(e));
    }
    {
        dbuf_status gs = step_grid_for(db->device, db->h_tiles.size(), &db->step_grid);
        if (gs != DBUF_OK) {
            delete db;
            return gs;
        }
        int sms = 1;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, db->device);
        const int64_t want = (db->plan.bucket / 8 + kNormThreads - 1) / kNormThreads;
        db->norm_grid = (int)std::max<int64_t>(1, std::min<int64_t>({want, (int64_t)kNormMaxCTAs, 4 * (int64_t)sms}));
    }
    if (device_base) {
        if ((reinterpret_cast<uintptr_t>(device_base) & 255u) != 0 || base_bytes < db->bytes) {
            const size_t need = db->bytes;
            delete db;
            return fail(DBUF_EINVAL, "dbuf_create: device_base must be 256-byte aligned and at least " +
                                         std::to_string(need) + " bytes");
        }
        db->base = static_cast<char*>(device_base);
        db->owns = false;
    } else {
        void* p = nullptr;
        e = cudaMalloc(&p, db->bytes);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            const size_t need = db->bytes;
            delete db;
            return fail(DBUF_ENOMEM, "dbuf_create: cudaMalloc of " + std::to_string(need) +
                                         " bytes failed: " + cudaGetErrorString(e));
        }
        db->base = static_cast<char*>(p);
        db->owns = true;
    }
    char* b = db->base;
    db->master = reinterpret_cast<float*>(b + db->lay.master);
    db->param = reinterpret_cast<uint16_t*>(b + db->lay.param);
    db->grad = reinterpret_cast<uint16_t*>(b + db->lay.grad);
    db->mq = reinterpret_cast<int8_t*>(b + db->lay.mq);
    db->vq = reinterpret_cast<uint8_t*>(b + db->lay.vq);
    db->scales = reinterpret_cast<float2*>(b + db->lay.scales);
    db->tiles = reinterpret_cast<Tile*>(b + db->lay.tiles);
    db->pos_tiles = reinterpret_cast<Tile*>(b + db->lay.pos_tiles);
    db->chunks = reinterpret_cast<PackChunk*>(b + db->lay.chunks);
    db->status = reinterpret_cast<int32_t*>(b + db->lay.status);
    db->scratch = reinterpret_cast<NormScratch*>(b + db->lay.scratch);
    e = cudaMemsetAsync(db->base, 0, db->bytes, st);
    if (e == cudaSuccess && !db->h_tiles.empty())
        e = cudaMemcpyAsync(db->tiles, db->h_tiles.data(), db->h_tiles.size() * sizeof(Tile),
                            cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess && !db->h_pos.tiles.empty())
        e = cudaMemcpyAsync(db->pos_tiles, db->h_pos.tiles.data(), db->h_pos.tiles.size() * sizeof(Tile),
                            cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess && !db->h_chunks.empty())
        e = cudaMemcpyAsync(db->chunks, db->h_chunks.data(), db->h_chunks.size() * sizeof(PackChunk),
                            cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess && db->h_host_chunks.size() > 1) {
        e = cudaStreamCreateWithFlags(&db->s_in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&db->s_out, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&db->ev_start, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&db->ev_done, cudaEventDisableTiming);
        db->ev_in.assign(db->h_host_chunks.size(), nullptr);
        db->ev_step.assign(db->h_host_chunks.size(), nullptr);
        for (size_t i = 0; e == cudaSuccess && i < db->h_host_chunks.size(); ++i) {
            e = cudaEventCreateWithFlags(&db->ev_in[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&db->ev_step[i], cudaEventDisableTiming);
        }
    }
    if (e != cudaSuccess) {
        release_pipeline(db);
        if (db->owns) cudaFree(db->base);
        delete db;
        return fail(DBUF_ECUDA, std::string("dbuf_create: initialising the bucket: ") + cudaGetErrorString(e));
    }
    *out = db;
    return DBUF_OK;
}

extern "C" void dbuf_destroy(dbuf_t* db) {
    if (!db) return;
    release_pipeline(db);
    if (db->owns && db->base) cudaFree(db->base);
    delete db;
}

static dbuf_status gather_grads(dbuf_t* db, const void* const* grads_bf16, float scale, void* stream, bool accumulate,
                                const char* who) {
    if (!db) return fail(DBUF_EINVAL, std::string(who) + ": db is NULL");
    if (db->plan.n > 0 && !grads_bf16) return fail(DBUF_EINVAL, std::string(who) + ": grads_bf16 is NULL");
    for (int32_t i = 0; i < db->plan.n; ++i)
        if (!grads_bf16[i] || (reinterpret_cast<uintptr_t>(grads_bf16[i]) & 1u))
            return fail(DBUF_EINVAL, std::string(who) + ": gradient pointer " + std::to_string(i) +
                                         " is NULL or not 2-byte aligned");
    dbuf_status s = check_device(db, who);
    if (s != DBUF_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t smem = kPackChunk * 2;
    for (int32_t t0 = 0; t0 < db->plan.n; t0 += kMaxPackPtrs) {
        const int32_t t1 = std::min<int32_t>(db->plan.n, t0 + kMaxPackPtrs);
        PackPtrs ptrs;
        std::memset(&ptrs, 0, sizeof ptrs);
        for (int32_t i = t0; i < t1; ++i) ptrs.p[i - t0] = static_cast<const uint16_t*>(grads_bf16[i]);
        const int64_t c0 = db->h_chunk_first[t0], c1 = db->h_chunk_first[t1];
        if (c1 <= c0) continue;
        if (accumulate)
            pack_kernel<true><<<(unsigned)(c1 - c0), kPackThreads, smem, st>>>(ptrs, db->chunks, c0, t0, db->grad,
                                                                                db->plan.bucket, scale, db->status);
        else
            pack_kernel<false><<<(unsigned)(c1 - c0), kPackThreads, smem, st>>>(ptrs, db->chunks, c0, t0, db->grad,
                                                                                 db->plan.bucket, scale, db->status);
        CUDA_TRY(cudaGetLastError(), who);
    }
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_pack_grads(dbuf_t* db, const void* const* grads_bf16, float scale, void* stream) {
    return gather_grads(db, grads_bf16, scale, stream, false, "dbuf_pack_grads");
}

extern "C" dbuf_status dbuf_accumulate_grads(dbuf_t* db, const void* const* grads_bf16, float scale, void* stream) {
    return gather_grads(db, grads_bf16, scale, stream, true, "dbuf_accumulate_grads");
}

static dbuf_status step_checks(dbuf_t* db, const dbuf_adam_hparams* hp, const char* who) {
    if (!db) return fail(DBUF_EINVAL, std::string(who) + ": db is NULL");
    if (!hp) return fail(DBUF_EINVAL, std::string(who) + ": hp is NULL");
    if (hp->step < 1) return fail(DBUF_EINVAL, std::string(who) + ": step must be >= 1");
    if (!(hp->beta1 >= 0.f && hp->beta1 < 1.f && hp->beta2 >= 0.f && hp->beta2 < 1.f))
        return fail(DBUF_EINVAL, std::string(who) + ": betas must be in [0, 1)");
    return check_device(db, who);
}

extern "C" dbuf_status dbuf_adam8_step(dbuf_t* db, const dbuf_adam_hparams* hp, float grad_scale, void* stream) {
    dbuf_status s = step_checks(db, hp, "dbuf_adam8_step");
    if (s != DBUF_OK) return s;
    if (db->h_tiles.empty()) return DBUF_OK;
    const StepC2 c = make_step_constants(*hp, grad_scale);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    adam8_step_kernel<<<(unsigned)db->step_grid, kStepThreads, kStepSmem, st>>>(
        db->tiles, (int64_t)db->h_tiles.size(), db->plan.bucket, db->master, db->param, db->grad, db->mq, db->vq,
        db->scales, db->plan.n_blocks, c, nullptr, db->status);
    CUDA_TRY(cudaGetLastError(), "dbuf_adam8_step: launch");
    return DBUF_OK;
}

static dbuf_status launch_norm(dbuf_t* db, float grad_scale, float max_norm, int clip, double* norm_dev,
                               cudaStream_t st, const char* who) {
    grad_norm_kernel<<<(unsigned)db->norm_grid, kNormThreads, 0, st>>>(db->grad, db->plan.bucket, grad_scale,
                                                                       max_norm, clip, db->scratch, norm_dev);
    CUDA_TRY(cudaGetLastError(), std::string(who) + ": norm launch");
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_grad_norm(dbuf_t* db, float grad_scale, double* norm_dev, void* stream) {
    if (!db) return fail(DBUF_EINVAL, "dbuf_grad_norm: db is NULL");
    if (!norm_dev) return fail(DBUF_EINVAL, "dbuf_grad_norm: norm_dev is NULL");
    dbuf_status s = check_device(db, "dbuf_grad_norm");
    if (s != DBUF_OK) return s;
    return launch_norm(db, grad_scale, 0.f, 0, norm_dev, reinterpret_cast<cudaStream_t>(stream), "dbuf_grad_norm");
}

// ------------------------------------------------ allocation-free norm
//
// For callers that cannot allocate device memory: code running where
// cudaMalloc is not allowed or not wanted (inside a custom allocator or a
// memory-pool callback, a runtime that owns every byte of device memory, a
// latency-critical loop that must not hit the allocator).  The norm
// reduction's scratch lives in this file-scope array instead: every GPU that
// loads the library holds it until the process exits.  One partial sum per
// CTA, one CTA per 2^20 elements, so one call covers at most 2^31 elements.

constexpr int64_t kNoAllocChunk = int64_t(1) << 20;
constexpr int64_t kNoAllocMaxElems = kNoAllocChunk * kNormMaxCTAs;  // 2^31

static __device__ __align__(256) NormScratch g_noalloc_norm_scratch;

namespace {
std::mutex g_noalloc_mu;
NormScratch* g_noalloc_ptr[256] = {nullptr};  // device address of the array, per device
}  // namespace

extern "C" dbuf_status dbuf_grad_norm_noalloc(const void* grad_bf16, int64_t n_elems, float grad_scale,
                                              double* norm_dev, void* stream) {
    const char* who = "dbuf_grad_norm_noalloc";
    if (n_elems < 0 || n_elems > kNoAllocMaxElems)
        return fail(DBUF_EINVAL, std::string(who) + ": n_elems must be in [0, 2^31] (the static scratch holds " +
                                     std::to_string(kNormMaxCTAs) + " partial sums of 2^20 elements each)");
    if (!norm_dev) return fail(DBUF_EINVAL, std::string(who) + ": norm_dev is NULL");
    if (n_elems > 0 && (!grad_bf16 || (reinterpret_cast<uintptr_t>(grad_bf16) & 15u)))
        return fail(DBUF_EINVAL, std::string(who) + ": grad_bf16 must be a 16-byte aligned device pointer");
    int dev = -1;
    CUDA_TRY(cudaGetDevice(&dev), who);
    if (dev < 0 || dev >= 256) return fail(DBUF_EINVAL, std::string(who) + ": device ordinal out of range");
    NormScratch* sc = nullptr;
    {
        // First call on a device: find the array's device address (host code
        // only holds a stand-in for it).
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (!g_noalloc_ptr[dev]) {
            void* p = nullptr;
            CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_norm_scratch), std::string(who) + ": scratch address");
            g_noalloc_ptr[dev] = static_cast<NormScratch*>(p);
        }
        sc = g_noalloc_ptr[dev];
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // The array keeps the last call's contents; the completion counter must
    // start at zero (a call that stopped early could have left it set).
    CUDA_TRY(cudaMemsetAsync(&sc->counter, 0, sizeof(uint32_t), st), std::string(who) + ": reset counter");
    const int grid = (int)std::max<int64_t>(1, (n_elems + kNoAllocChunk - 1) / kNoAllocChunk);
    grad_norm_kernel<<<(unsigned)grid, kNormThreads, 0, st>>>(static_cast<const uint16_t*>(grad_bf16), n_elems,
                                                              grad_scale, 0.f, 0, sc, norm_dev);
    CUDA_TRY(cudaGetLastError(), std::string(who) + ": launch");
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_adam8_step_clipped(dbuf_t* db, const dbuf_adam_hparams* hp, float grad_scale,
                                               float max_norm, double* norm_dev, void* stream) {
    dbuf_status s = step_checks(db, hp, "dbuf_adam8_step_clipped");
    if (s != DBUF_OK) return s;
    if (!(max_norm > 0.f)) return fail(DBUF_EINVAL, "dbuf_adam8_step_clipped: max_norm must be > 0");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    s = launch_norm(db, grad_scale, max_norm, 1, norm_dev, st, "dbuf_adam8_step_clipped");
    if (s != DBUF_OK) return s;
    if (db->h_tiles.empty()) return DBUF_OK;
    const StepC2 c = make_step_constants(*hp, grad_scale);
    adam8_step_kernel<<<(unsigned)db->step_grid, kStepThreads, kStepSmem, st>>>(
        db->tiles, (int64_t)db->h_tiles.size(), db->plan.bucket, db->master, db->param, db->grad, db->mq, db->vq,
        db->scales, db->plan.n_blocks, c, &db->scratch->gscale_eff, db->status);
    CUDA_TRY(cudaGetLastError(), "dbuf_adam8_step_clipped: launch");
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_adam8_step_host(dbuf_t* db, const dbuf_adam_hparams* hp, float grad_scale,
                                            const void* grads_host, void* params_bf16_host, void* stream) {
    dbuf_status s = step_checks(db, hp, "dbuf_adam8_step_host");
    if (s != DBUF_OK) return s;
    if (db->plan.bucket > 0 && (!grads_host || !params_bf16_host))
        return fail(DBUF_EINVAL, "dbuf_adam8_step_host: host buffer is NULL");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t bytes = (size_t)db->plan.bucket * 2;
    if (db->h_host_chunks.size() <= 1) {
        if (bytes) CUDA_TRY(cudaMemcpyAsync(db->grad, grads_host, bytes, cudaMemcpyHostToDevice, st),
                            "dbuf_adam8_step_host: copy in");
        s = dbuf_adam8_step(db, hp, grad_scale, stream);
        if (s != DBUF_OK) return s;
        if (bytes) CUDA_TRY(cudaMemcpyAsync(params_bf16_host, db->param, bytes, cudaMemcpyDeviceToHost, st),
                            "dbuf_adam8_step_host: copy out");
        return DBUF_OK;
    }
    // Chunked pipeline: chunk i's gradients arrive on s_in, its entries are
    // stepped on `stream` once they have, and its bf16 params leave on s_out
    // once stepped, so the two copy directions and the step overlap.  The
    // chunks' element ranges partition the bucket and every entry reads and
    // writes inside its chunk's range (a bulk copy may also read up to 15
    // elements beyond it, into lanes the step ignores).
    const StepC2 c = make_step_constants(*hp, grad_scale);
    const char* gh = static_cast<const char*>(grads_host);
    char* ph = static_cast<char*>(params_bf16_host);
    CUDA_TRY(cudaEventRecord(db->ev_start, st), "dbuf_adam8_step_host: record");
    CUDA_TRY(cudaStreamWaitEvent(db->s_in, db->ev_start, 0), "dbuf_adam8_step_host: wait");
    CUDA_TRY(cudaStreamWaitEvent(db->s_out, db->ev_start, 0), "dbuf_adam8_step_host: wait");
    for (size_t i = 0; i < db->h_host_chunks.size(); ++i) {
        const HostChunk& hc = db->h_host_chunks[i];
        const size_t off = (size_t)hc.lo * 2, len = (size_t)(hc.hi - hc.lo) * 2;
        CUDA_TRY(cudaMemcpyAsync(reinterpret_cast<char*>(db->grad) + off, gh + off, len, cudaMemcpyHostToDevice,
                                 db->s_in),
                 "dbuf_adam8_step_host: copy in");
        CUDA_TRY(cudaEventRecord(db->ev_in[i], db->s_in), "dbuf_adam8_step_host: record");
        CUDA_TRY(cudaStreamWaitEvent(st, db->ev_in[i], 0), "dbuf_adam8_step_host: wait");
        const int64_t nt = hc.t1 - hc.t0;
        adam8_step_kernel<<<(unsigned)std::min<int64_t>(nt, db->step_grid), kStepThreads, kStepSmem, st>>>(
            db->pos_tiles + hc.t0, nt, db->plan.bucket, db->master, db->param, db->grad, db->mq, db->vq,
            db->scales, db->plan.n_blocks, c, nullptr, db->status);
        CUDA_TRY(cudaGetLastError(), "dbuf_adam8_step_host: launch");
        CUDA_TRY(cudaEventRecord(db->ev_step[i], st), "dbuf_adam8_step_host: record");
        CUDA_TRY(cudaStreamWaitEvent(db->s_out, db->ev_step[i], 0), "dbuf_adam8_step_host: wait");
        CUDA_TRY(cudaMemcpyAsync(ph + off, reinterpret_cast<const char*>(db->param) + off, len,
                                 cudaMemcpyDeviceToHost, db->s_out),
                 "dbuf_adam8_step_host: copy out");
    }
    CUDA_TRY(cudaEventRecord(db->ev_done, db->s_out), "dbuf_adam8_step_host: record");
    CUDA_TRY(cudaStreamWaitEvent(st, db->ev_done, 0), "dbuf_adam8_step_host: wait");
    return DBUF_OK;
}

static void* array_of(const dbuf_t* db, dbuf_which w, size_t* esize) {
    switch (w) {
        case DBUF_MASTER_F32: *esize = 4; return db->master;
        case DBUF_PARAM_BF16: *esize = 2; return db->param;
        case DBUF_GRAD_BF16: *esize = 2; return db->grad;
        case DBUF_M_I8: *esize = 1; return db->mq;
        case DBUF_V_U8: *esize = 1; return db->vq;
    }
    return nullptr;
}

extern "C" dbuf_status dbuf_unpack_views(const dbuf_t* db, dbuf_which which, dbuf_view* out) {
    if (!db) return fail(DBUF_EINVAL, "dbuf_unpack_views: db is NULL");
    size_t es = 0;
    char* a = static_cast<char*>(array_of(db, which, &es));
    if (!a) return fail(DBUF_EINVAL, "dbuf_unpack_views: unknown array kind");
    if (db->plan.n > 0 && !out) return fail(DBUF_EINVAL, "dbuf_unpack_views: out is NULL");
    for (int32_t i = 0; i < db->plan.n; ++i)
        out[i] = dbuf_view{a + (size_t)db->plan.offset[i] * es, db->plan.rows[i], db->plan.cols[i], db->plan.offset[i]};
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_bucket(const dbuf_t* db, dbuf_which which, void** ptr, int64_t* elems) {
    if (!db) return fail(DBUF_EINVAL, "dbuf_bucket: db is NULL");
    size_t es = 0;
    void* a = array_of(db, which, &es);
    if (!a) return fail(DBUF_EINVAL, "dbuf_bucket: unknown array kind");
    if (ptr) *ptr = a;
    if (elems) *elems = db->plan.bucket;
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_scales(const dbuf_t* db, float** scales, int64_t* n_blocks) {
    if (!db) return fail(DBUF_EINVAL, "dbuf_scales: db is NULL");
    if (scales) *scales = reinterpret_cast<float*>(db->scales);
    if (n_blocks) *n_blocks = db->plan.n_blocks;
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_get_device_status(dbuf_t* db, int32_t* code, void* stream) {
    if (!db || !code) return fail(DBUF_EINVAL, "dbuf_get_device_status: NULL argument");
    dbuf_status s = check_device(db, "dbuf_get_device_status");
    if (s != DBUF_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t h = 0;
    CUDA_TRY(cudaMemcpyAsync(&h, db->status, sizeof h, cudaMemcpyDeviceToHost, st), "dbuf_get_device_status");
    CUDA_TRY(cudaStreamSynchronize(st), "dbuf_get_device_status: sync");
    *code = h;
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_clear_device_status(dbuf_t* db, void* stream) {
    if (!db) return fail(DBUF_EINVAL, "dbuf_clear_device_status: db is NULL");
    dbuf_status s = check_device(db, "dbuf_clear_device_status");
    if (s != DBUF_OK) return s;
    CUDA_TRY(cudaMemsetAsync(db->status, 0, sizeof(int32_t), reinterpret_cast<cudaStream_t>(stream)),
             "dbuf_clear_device_status");
    CUDA_TRY(cudaMemsetAsync(&db->scratch->counter, 0, sizeof(uint32_t), reinterpret_cast<cudaStream_t>(stream)),
             "dbuf_clear_device_status: norm counter");
    return DBUF_OK;
}
