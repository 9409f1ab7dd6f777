// Plain CPU oracle of the ragged-bucket 8-bit Adam step.
//
// TEST INFRASTRUCTURE ONLY: tests, the smoke check and the bench's CPU
// baseline call this; the product library never does, and this file shares
// no code, header, table or helper with it.
//
// What it follows (veScale-FSDP, MLSys 2026, as summarised on the gist.science
// and notes.yuuk.io pages; "Sec." numbers are the paper sections those pages
// attribute each statement to):
//   * RaggedShard (Sec. 3): every tensor is cut into whole blocks of k rows;
//     a block is never split between two devices, devices may hold different
//     numbers of blocks.
//   * Structure-aware planning (Sec. 4): tensors are sorted by block size,
//     largest first, then a dynamic program chooses placement offsets inside
//     the communication bucket; padding goes between tensors, never inside
//     one, and the bucket is cut into m equal per-device slices.
//   * DBuffer (Sec. 5): the bucket is one flat buffer, tensors are views.
//   * 8-bit Adam case study (Sec. 6.3): block-wise quantised optimizer states,
//     each device quantising its own blocks without communication, with
//     blocks of k whole rows or 2-D tiles (e.g. 32x32 elements) per
//     parameter; a tile is gathered and stepped as one block.
// The pages give no formulas for the quantiser or the update; the readings
// taken here (linear absmax codes, int8 m, uint8 sqrt(v), decoupled weight
// decay, round-half-even) are listed in the project's design notes.
//
// Precision: the update is plain IEEE fp32 in one fixed operation order,
// built with -ffp-contract=off and without fast-math, so every product and
// sum is rounded on its own.  Per-step scalars are formed in double and
// rounded to float once.
//
// Parity status: layout and update are pinned by the CPU tests (literal
// definition scans, exhaustive search on tiny instances, the closed-form first
// step, code invariants, an fp64 shadow); the 2-D tile step by a worked first
// step and by equality with the contiguous step on cut-out tiles.  The rank
// buckets (rank_bucket in __init__.py: one slice as a bucket of its own) are
// pinned by stepping every rank's bucket alone and finding the whole bucket's
// result bit for bit, and by their parts tiling every tensor.  Parity with
// the pages' own system is unpinned: the pages print no worked example.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <vector>

namespace {

struct T {
    int64_t n;  // elements
    int64_t b;  // block size in elements (k * cols)
    int64_t idx;
};

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t q) { return ceil_div(a, q) * q; }

// The layout rule in words: a start o is allowed for a tensor of n elements
// and block size b iff o is a multiple of the alignment A, the tensor ends
// inside the bucket (o + n <= m*s), and every slice boundary r*s strictly
// inside the tensor falls on one of its block edges ((r*s - o) % b == 0).
bool start_allowed(int64_t o, int64_t n, int64_t b, int64_t s, int64_t m, int64_t A) {
    if (o % A != 0) return false;
    if (o + n > m * s) return false;
    // Boundaries at or before o are not inside; start from the first after it.
    for (int64_t r = o / s + 1; r < m && r * s < o + n; ++r)
        if ((r * s - o) % b != 0) return false;
    return true;
}

// Earliest allowed start >= lo, by scanning every multiple of A.  Exactly the
// definition; far too slow for real buckets, used on small ones to check the
// walk below.
int64_t earliest_literal(int64_t lo, int64_t n, int64_t b, int64_t s, int64_t m, int64_t A) {
    for (int64_t o = round_up(lo, A); o + n <= m * s; o += A)
        if (start_allowed(o, n, b, s, m, A)) return o;
    return -1;
}

// Earliest allowed start >= lo, walking slice by slice.
//  * If the tensor fits in the rest of the current slice, the first aligned
//    position is allowed.
//  * Otherwise every start left in this slice has the next boundary R inside
//    the tensor, so it must satisfy (R - o) % b == 0 and o % A == 0, i.e.
//    R - o is a positive multiple of lcm(A, b).  The smallest such o is the
//    only one worth checking: any later o in this slice sees the same or more
//    boundaries inside the tensor, each with the same residue, and ends later.
//  * If that candidate is not allowed, continue at the next slice start.
int64_t earliest_walk(int64_t lo, int64_t n, int64_t b, int64_t s, int64_t m, int64_t A) {
    int64_t o = round_up(lo, A);
    const int64_t L = std::lcm(A, b);
    while (o + n <= m * s) {
        int64_t R = (o / s + 1) * s;
        if (o + n <= R) return o;
        int64_t j = ((R - o) / L) * L;
        if (j > 0 && start_allowed(R - j, n, b, s, m, A)) return R - j;
        o = R;
    }
    return -1;
}

// Sort key of the planner: block size descending (the pages' heuristic);
// ties broken by element count descending, then by input position.
std::vector<T> sorted_tensors(const int64_t* rows, const int64_t* cols, const int64_t* k, int32_t n) {
    std::vector<T> ts(n);
    for (int32_t i = 0; i < n; ++i) ts[i] = T{rows[i] * cols[i], k[i] * cols[i], i};
    std::sort(ts.begin(), ts.end(), [](const T& x, const T& y) {
        if (x.b != y.b) return x.b > y.b;
        if (x.n != y.n) return x.n > y.n;
        return x.idx < y.idx;
    });
    return ts;
}

// Greedy placement in the fixed order.  For a fixed order and slice size this
// is the dynamic program over offsets with its state collapsed: the set of
// allowed starts of each tensor does not depend on earlier tensors, and an
// earlier end never removes a later option, so taking the earliest allowed
// start for every tensor is optimal (checked by exhaustive search in tests).
bool place_all(const std::vector<T>& ts, int64_t s, int64_t m, int64_t A, bool literal, int64_t* off) {
    int64_t end = 0;
    for (const T& t : ts) {
        int64_t o = literal ? earliest_literal(end, t.n, t.b, s, m, A)
                            : earliest_walk(end, t.n, t.b, s, m, A);
        if (o < 0) return false;
        off[t.idx] = o;
        end = o + t.n;
    }
    return true;
}

// A tensor longer than 2s always has two consecutive slice boundaries inside
// it, both on block edges, so its block size must divide s.  Slice sizes that
// break this are skipped without running the placement (they would fail it).
bool necessary_ok(const std::vector<T>& ts, int64_t s) {
    for (const T& t : ts)
        if (t.n > 2 * s && s % t.b != 0) return false;
    return true;
}

}  // namespace

extern "C" {

// Status codes of the oracle entry points.
enum { ORC_OK = 0, ORC_EINVAL = 1, ORC_EINFEASIBLE = 2 };

// Plan a bucket.  offsets[i] receives the start of input tensor i; *slice the
// slice size s (bucket = m*s).  literal=1 uses the definition scan and no
// skipping (tiny inputs only).  max_bucket=0 means no cap.
int orc_plan(const int64_t* rows, const int64_t* cols, const int64_t* k, int32_t n, int32_t m,
             int64_t A, int64_t max_bucket, int32_t literal, int64_t* offsets, int64_t* slice) {
    if (n < 0 || m < 1 || A < 1) return ORC_EINVAL;
    for (int32_t i = 0; i < n; ++i)
        if (rows[i] < 1 || cols[i] < 1 || k[i] < 1 || k[i] > rows[i]) return ORC_EINVAL;
    std::vector<T> ts = sorted_tensors(rows, cols, k, n);
    int64_t total = 0, upper = 0;
    for (const T& t : ts) {
        total += t.n;
        upper += round_up(t.n, A);
    }
    // s = 0 holds an empty bucket; otherwise start at the even share.
    int64_t s = round_up(ceil_div(total, m), A);
    upper = round_up(upper, A);  // everything fits in slice 0 at this size
    for (; s <= upper; s += A) {
        if (max_bucket > 0 && s * (int64_t)m > max_bucket) return ORC_EINFEASIBLE;
        if (s == 0) {
            *slice = 0;
            return ORC_OK;
        }
        if (!literal && !necessary_ok(ts, s)) continue;
        if (place_all(ts, s, m, A, literal != 0, offsets)) {
            *slice = s;
            return ORC_OK;
        }
    }
    return ORC_EINFEASIBLE;  // not reached: s = upper always places
}

// Greedy placement at one fixed slice size s (no search over s): 1 if every
// tensor got a start, 0 otherwise.  offsets as in orc_plan.
int orc_place_fixed(const int64_t* rows, const int64_t* cols, const int64_t* k, int32_t n, int32_t m,
                    int64_t A, int64_t s, int32_t literal, int64_t* offsets) {
    if (s <= 0) return n == 0 ? 1 : 0;
    std::vector<T> ts = sorted_tensors(rows, cols, k, n);
    return place_all(ts, s, m, A, literal != 0, offsets) ? 1 : 0;
}

// Is there ANY placement of the tensors, in the given order, at slice size s?
// Exhaustive depth-first search over every allowed start (tiny inputs only).
static bool dfs(const int64_t* n, const int64_t* b, int32_t cnt, int32_t i, int64_t end, int64_t s,
                int64_t m, int64_t A) {
    if (i == cnt) return true;
    for (int64_t o = round_up(end, A); o + n[i] <= m * s; o += A)
        if (start_allowed(o, n[i], b[i], s, m, A) && dfs(n, b, cnt, i + 1, o + n[i], s, m, A))
            return true;
    return false;
}

int orc_exists_placement(const int64_t* n, const int64_t* b, int32_t cnt, int64_t s, int32_t m,
                         int64_t A) {
    return dfs(n, b, cnt, 0, 0, s, m, A) ? 1 : 0;
}

// Smallest bucket (m*s) over EVERY order of the tensors and every placement:
// the true minimum padding.  Exponential; for at most ~6 tiny tensors.
int64_t orc_bruteforce_min_bucket(const int64_t* rows, const int64_t* cols, const int64_t* k,
                                  int32_t cnt, int32_t m, int64_t A) {
    std::vector<int32_t> perm(cnt);
    std::iota(perm.begin(), perm.end(), 0);
    int64_t total = 0, upper = 0;
    for (int32_t i = 0; i < cnt; ++i) {
        total += rows[i] * cols[i];
        upper += round_up(rows[i] * cols[i], A);
    }
    upper = round_up(upper, A);
    int64_t best = -1;
    std::vector<int64_t> n(cnt), b(cnt);
    do {
        for (int32_t i = 0; i < cnt; ++i) {
            n[i] = rows[perm[i]] * cols[perm[i]];
            b[i] = k[perm[i]] * cols[perm[i]];
        }
        for (int64_t s = round_up(ceil_div(total, m), A); s <= upper; s += A) {
            if (best >= 0 && s * m >= best) break;
            if (s == 0 || dfs(n.data(), b.data(), cnt, 0, 0, s, m, A)) {
                best = s * m;
                break;
            }
        }
    } while (std::next_permutation(perm.begin(), perm.end()));
    return best;
}

// Layout checker.  Returns a bit mask of broken rules (0 = valid):
//   1  slice size not a multiple of A, or below the even share
//   2  a start not a multiple of A
//   4  a tensor outside [0, m*s)
//   8  two tensors overlap
//  16  a slice boundary inside a tensor off its block edges
int orc_check_layout(const int64_t* rows, const int64_t* cols, const int64_t* k, int32_t n,
                     int32_t m, int64_t A, const int64_t* off, int64_t s) {
    int bad = 0;
    int64_t total = 0;
    for (int32_t i = 0; i < n; ++i) total += rows[i] * cols[i];
    if (s < 0 || s % A != 0 || s * m < total) bad |= 1;
    std::vector<std::pair<int64_t, int64_t>> iv;
    for (int32_t i = 0; i < n; ++i) {
        int64_t len = rows[i] * cols[i], b = k[i] * cols[i];
        if (off[i] % A != 0) bad |= 2;
        if (off[i] < 0 || off[i] + len > s * m) bad |= 4;
        for (int64_t r = 1; r < m; ++r) {
            int64_t R = r * s;
            if (off[i] < R && R < off[i] + len && (R - off[i]) % b != 0) bad |= 16;
        }
        iv.push_back({off[i], off[i] + len});
    }
    std::sort(iv.begin(), iv.end());
    for (size_t i = 1; i < iv.size(); ++i)
        if (iv[i].first < iv[i - 1].second) bad |= 8;
    return bad;
}

// Round a float to bfloat16, nearest with ties to even (NaN kept quiet).
static uint16_t bf16_rne(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static float bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

// Per-step scalars of Adam with bias correction and decoupled weight decay,
// formed in double from the float hyper-parameters, rounded to float once.
// The bias corrections are folded into the step size and eps, as the
// published 8-bit optimizers do (Dettmers et al., "8-bit Optimizers via
// Block-wise Quantization", ICLR 2022):
//   (lr / bc1) * m / (sqrt(v) / sqrt(bc2) + eps)
//     = (lr * sqrt(bc2) / bc1) * m / (sqrt(v) + eps * sqrt(bc2)),
// with bc1 = 1 - b1^t, bc2 = 1 - b2^t: one division per element.
struct Scalars {
    float b1, omb1, b2, omb2, sqrt_bc2, eps_hat, step_hat, decay;
};

static Scalars make_scalars(float lr, float beta1, float beta2, float eps, float wd, int64_t t) {
    double l = lr, B1 = beta1, B2 = beta2, E = eps, W = wd;
    double bc1 = 1.0 - std::pow(B1, (double)t);
    double sq2 = std::sqrt(1.0 - std::pow(B2, (double)t));
    Scalars c;
    c.b1 = (float)B1;
    c.omb1 = (float)(1.0 - B1);
    c.b2 = (float)B2;
    c.omb2 = (float)(1.0 - B2);
    c.sqrt_bc2 = (float)sq2;
    c.eps_hat = (float)(E * sq2);
    c.step_hat = (float)(l * sq2 / bc1);
    c.decay = (float)(1.0 - l * W);
    return c;
}

// One block of block-wise 8-bit Adam, in place.
//   p      fp32 master weights of the block (len elements)
//   g      bf16 gradient bits
//   mq     int8 codes of m, vq uint8 codes of sqrt(v)
//   sm,sv  the block's scales (absmax of m and of sqrt(v) at the last step)
//   pb     bf16 copy of the updated weights
// The state a code stands for is code * scale / 127 (m) and
// (code * scale / 255)^2 (v).  The update uses the unquantised new m and v;
// only what is stored is quantised.
static void adam8_block(int64_t len, float* p, const uint16_t* g, int8_t* mq, uint8_t* vq, float* sm,
                        float* sv, uint16_t* pb, const Scalars& c, float grad_scale, float* mt,
                        float* rt) {
    const float dqm = *sm / 127.0f;
    const float dqv = *sv / 255.0f;
    float amax_m = 0.0f, amax_r = 0.0f;
    for (int64_t i = 0; i < len; ++i) {
        float gi = bf16_to_f32(g[i]) * grad_scale;
        float mo = (float)mq[i] * dqm;
        float so = (float)vq[i] * dqv;
        float vo = so * so;
        float m = c.b1 * mo;
        float t = c.omb1 * gi;
        m = m + t;
        float v = c.b2 * vo;
        float gg = gi * gi;
        t = c.omb2 * gg;
        v = v + t;
        float r = std::sqrt(v);
        float d = r + c.eps_hat;
        float u = m / d;
        float pn = p[i] * c.decay;
        t = c.step_hat * u;
        pn = pn - t;
        p[i] = pn;
        pb[i] = bf16_rne(pn);
        mt[i] = m;
        rt[i] = r;
        amax_m = std::max(amax_m, std::fabs(m));
        amax_r = std::max(amax_r, r);
    }
    // Requantise with the block's new absmax.
    const float qm = amax_m > 0.0f ? 127.0f / amax_m : 0.0f;
    const float qv = amax_r > 0.0f ? 255.0f / amax_r : 0.0f;
    for (int64_t i = 0; i < len; ++i) {
        float a = std::rint(mt[i] * qm);
        float b = std::rint(rt[i] * qv);
        a = std::min(127.0f, std::max(-127.0f, a));
        b = std::min(255.0f, std::max(0.0f, b));
        mq[i] = (int8_t)a;
        vq[i] = (uint8_t)b;
    }
    *sm = amax_m;
    *sv = amax_r;
}

// Step a list of blocks.  Block j covers bucket elements
// [start[j], start[j] + len[j]) and owns scales scale_m[sidx[j]], scale_v[sidx[j]].
// threads > 1 splits the block list over OpenMP threads; every block is
// computed by the same function either way, so results do not depend on it.
void orc_adam8_step(int64_t n_blocks, const int64_t* start, const int64_t* len, const int64_t* sidx,
                    float* p, const uint16_t* g, int8_t* mq, uint8_t* vq, float* scale_m,
                    float* scale_v, uint16_t* pb, float lr, float beta1, float beta2, float eps,
                    float wd, int64_t step, float grad_scale, int32_t threads) {
    const Scalars c = make_scalars(lr, beta1, beta2, eps, wd, step);
    int64_t maxlen = 0;
    for (int64_t j = 0; j < n_blocks; ++j) maxlen = std::max(maxlen, len[j]);
#pragma omp parallel num_threads(threads > 0 ? threads : 1) if (threads > 1)
    {
        std::vector<float> mt(maxlen > 0 ? maxlen : 1), rt(maxlen > 0 ? maxlen : 1);
#pragma omp for schedule(dynamic, 16)
        for (int64_t j = 0; j < n_blocks; ++j) {
            int64_t o = start[j];
            adam8_block(len[j], p + o, g + o, mq + o, vq + o, scale_m + sidx[j], scale_v + sidx[j],
                        pb + o, c, grad_scale, mt.data(), rt.data());
        }
    }
}

// Step a list of 2-D tiles (the 32x32-element blocks of the 8-bit Adam case
// study: a block of trows[j] rows and width[j] columns of a row-major tensor
// whose rows are stride[j] elements apart).  Tile j covers the elements
// base[j] + r * stride[j] + c, r < trows[j], c < width[j], and owns scales
// scale_m[sidx[j]], scale_v[sidx[j]].  Its elements are gathered in row-major
// order, stepped as one block by adam8_block, and written back.
void orc_adam8_step_tiles(int64_t n_tiles, const int64_t* base, const int64_t* trows, const int64_t* width,
                          const int64_t* stride, const int64_t* sidx, float* p, const uint16_t* g, int8_t* mq,
                          uint8_t* vq, float* scale_m, float* scale_v, uint16_t* pb, float lr, float beta1,
                          float beta2, float eps, float wd, int64_t step, float grad_scale, int32_t threads) {
    const Scalars c = make_scalars(lr, beta1, beta2, eps, wd, step);
    int64_t maxlen = 0;
    for (int64_t j = 0; j < n_tiles; ++j) maxlen = std::max(maxlen, trows[j] * width[j]);
    const size_t L = (size_t)(maxlen > 0 ? maxlen : 1);
#pragma omp parallel num_threads(threads > 0 ? threads : 1) if (threads > 1)
    {
        std::vector<float> mt(L), rt(L), tp(L);
        std::vector<uint16_t> tg(L), tpb(L);
        std::vector<int8_t> tm(L);
        std::vector<uint8_t> tv(L);
        std::vector<int64_t> at(L);
#pragma omp for schedule(dynamic, 16)
        for (int64_t j = 0; j < n_tiles; ++j) {
            const int64_t n = trows[j] * width[j];
            for (int64_t r = 0; r < trows[j]; ++r)
                for (int64_t q = 0; q < width[j]; ++q) at[r * width[j] + q] = base[j] + r * stride[j] + q;
            for (int64_t i = 0; i < n; ++i) {
                tp[i] = p[at[i]];
                tg[i] = g[at[i]];
                tm[i] = mq[at[i]];
                tv[i] = vq[at[i]];
            }
            adam8_block(n, tp.data(), tg.data(), tm.data(), tv.data(), scale_m + sidx[j], scale_v + sidx[j],
                        tpb.data(), c, grad_scale, mt.data(), rt.data());
            for (int64_t i = 0; i < n; ++i) {
                p[at[i]] = tp[i];
                mq[at[i]] = tm[i];
                vq[at[i]] = tv[i];
                pb[at[i]] = tpb[i];
            }
        }
    }
}

// The per-step scalars as floats, in the order b1, omb1, b2, omb2, sqrt_bc2,
// eps_hat, step_hat, decay (for the tests' closed forms).
void orc_step_scalars(float lr, float beta1, float beta2, float eps, float wd, int64_t t, float* out) {
    Scalars c = make_scalars(lr, beta1, beta2, eps, wd, t);
    float v[8] = {c.b1, c.omb1, c.b2, c.omb2, c.sqrt_bc2, c.eps_hat, c.step_hat, c.decay};
    std::memcpy(out, v, sizeof v);
}

// Copy-in gather of the row-wise FSDP baseline: one tensor's gradient into
// its planned place in the bucket, scaled: dst[i] = bf16(float(src[i]) * scale).
void orc_pack(int64_t count, const uint16_t* src, uint16_t* dst, float scale) {
    for (int64_t i = 0; i < count; ++i) dst[i] = bf16_rne(bf16_to_f32(src[i]) * scale);
}

// DBuffer group "add" (gradient accumulation across micro-batches): one
// tensor's gradient added into its place in the bucket,
//   dst[i] = bf16(float(dst[i]) + float(src[i]) * scale).
void orc_accumulate(int64_t count, const uint16_t* src, uint16_t* dst, float scale) {
    for (int64_t i = 0; i < count; ++i) {
        float t = bf16_to_f32(src[i]) * scale;
        float s = bf16_to_f32(dst[i]) + t;
        dst[i] = bf16_rne(s);
    }
}

// Global L2 norm of the scaled gradient bucket: each element is scaled in
// fp32 exactly as the step does, squared and summed in double, in order.
double orc_grad_norm(int64_t count, const uint16_t* g, float scale) {
    double acc = 0.0;
    for (int64_t i = 0; i < count; ++i) {
        double x = (double)(bf16_to_f32(g[i]) * scale);
        acc += x * x;
    }
    return std::sqrt(acc);
}

// Gradient scale after global-norm clipping (the convention of
// torch.nn.utils.clip_grad_norm_: coefficient max_norm / (norm + 1e-6),
// applied only when below 1), folded into the step's grad_scale in double
// and rounded to float once.
double orc_clip_coef(double norm, float max_norm) {
    double coef = (double)max_norm / (norm + 1e-6);
    return coef < 1.0 ? coef : 1.0;
}

float orc_clipped_scale(double norm, float grad_scale, float max_norm) {
    double coef = orc_clip_coef(norm, max_norm);
    if (coef >= 1.0) return grad_scale;
    return (float)((double)grad_scale * coef);
}

// bf16 rounding on its own, for the tests.
void orc_bf16_round(int64_t count, const float* x, uint16_t* out) {
    for (int64_t i = 0; i < count; ++i) out[i] = bf16_rne(x[i]);
}

}  // extern "C"
