// Distributed Muon on the bucket (the C-ABI's dbuf_muon_* functions):
// momentum and normalisation in our kernels (muon_kernels.cuh), the
// Newton-Schulz iteration as cuBLAS GEMMs (bf16 operands, fp32
// accumulation, tensor cores), the weight update in our kernel.  The pages'
// case study ("8-bit Adam and distributed Muon", paper Sec. 6.3) gathers each
// 2-D parameter whole on one rank; in a bucket each tensor is already whole,
// so the state works on the tensor's own views.
#include <cublas_v2.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <new>
#include <string>
#include <vector>

#include "internal.h"
#include "muon_kernels.cuh"

using dbuf_detail::fail;
using namespace dbuf_k;

namespace {

// Coefficients of the quintic Newton-Schulz step (Muon, K. Jordan et al.).
constexpr float kNsA = 3.4445f, kNsB = -4.7750f, kNsC = 2.0315f;

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

struct dbuf_muon_s {
    dbuf_t* db = nullptr;
    int device = -1;
    std::vector<int32_t> ids;
    std::vector<int64_t> rows, cols, mom_off;
    std::vector<float*> master;
    std::vector<uint16_t*> param, grad;
    int64_t cap_rc = 0, cap_ss = 0;
    char* base = nullptr;
    float* mom = nullptr;
    float* u = nullptr;               // fp32 direction, cap_rc
    __nv_bfloat16* x = nullptr;       // iterate, cap_rc
    __nv_bfloat16* y = nullptr;       // next iterate, cap_rc
    __nv_bfloat16* a = nullptr;       // X X^T, cap_ss
    __nv_bfloat16* b = nullptr;       // b A + c A A, cap_ss
    double* partial = nullptr;        // kMuonMaxCTAs
    cublasHandle_t h = nullptr;
};

#define CUBLAS_TRY(call, what)                                                                 \
    do {                                                                                       \
        cublasStatus_t s_ = (call);                                                            \
        if (s_ != CUBLAS_STATUS_SUCCESS)                                                       \
            return fail(DBUF_ECUDA, std::string(what) + ": cuBLAS status " + std::to_string((int)s_)); \
    } while (0)

static int muon_grid(int64_t n) {
    const int64_t want = (n + kMuonThreads * 8 - 1) / (kMuonThreads * 8);
    return (int)std::max<int64_t>(1, std::min<int64_t>(want, kMuonMaxCTAs));
}

extern "C" void dbuf_muon_destroy(dbuf_muon_t* mu) {
    if (!mu) return;
    if (mu->h) cublasDestroy(mu->h);
    if (mu->base) cudaFree(mu->base);
    delete mu;
}

extern "C" dbuf_status dbuf_muon_create(dbuf_t* db, const int32_t* ids, int32_t n, void* stream, dbuf_muon_t** out) {
    if (!out) return fail(DBUF_EINVAL, "dbuf_muon_create: out is NULL");
    *out = nullptr;
    if (!db || !ids || n < 1) return fail(DBUF_EINVAL, "dbuf_muon_create: need a dbuf and n >= 1 tensor ids");
    const int32_t nt = dbuf_detail::tensors_of(db);
    int dev = -1;
    CUDA_TRY(cudaGetDevice(&dev), "dbuf_muon_create");
    if (dev != dbuf_detail::device_of(db)) return fail(DBUF_EINVAL, "dbuf_muon_create: wrong current device");
    std::vector<dbuf_view> vm(nt), vp(nt), vg(nt);
    dbuf_status st = dbuf_unpack_views(db, DBUF_MASTER_F32, vm.data());
    if (st == DBUF_OK) st = dbuf_unpack_views(db, DBUF_PARAM_BF16, vp.data());
    if (st == DBUF_OK) st = dbuf_unpack_views(db, DBUF_GRAD_BF16, vg.data());
    if (st != DBUF_OK) return st;
    dbuf_muon_s* mu = new (std::nothrow) dbuf_muon_s;
    if (!mu) return fail(DBUF_ENOMEM, "dbuf_muon_create: out of host memory");
    mu->db = db;
    mu->device = dev;
    std::vector<char> used(nt, 0);
    int64_t total = 0;
    for (int32_t j = 0; j < n; ++j) {
        const int32_t i = ids[j];
        if (i < 0 || i >= nt || used[i] || vm[i].rows < 2 || vm[i].cols < 2) {
            delete mu;
            return fail(DBUF_EINVAL, "dbuf_muon_create: id " + std::to_string(i) +
                                         " is out of range, repeated, or not a 2-D tensor with rows, cols >= 2");
        }
        used[i] = 1;
        const int64_t R = vm[i].rows, C = vm[i].cols, s = std::min(R, C);
        mu->ids.push_back(i);
        mu->rows.push_back(R);
        mu->cols.push_back(C);
        mu->mom_off.push_back(total);
        mu->master.push_back(static_cast<float*>(vm[i].ptr));
        mu->param.push_back(static_cast<uint16_t*>(vp[i].ptr));
        mu->grad.push_back(static_cast<uint16_t*>(vg[i].ptr));
        total += R * C;
        mu->cap_rc = std::max(mu->cap_rc, R * C);
        mu->cap_ss = std::max(mu->cap_ss, s * s);
    }
    const size_t b_mom = up256((size_t)total * 4), b_u = up256((size_t)mu->cap_rc * 4),
                 b_x = up256((size_t)mu->cap_rc * 2), b_a = up256((size_t)mu->cap_ss * 2),
                 b_p = up256((size_t)kMuonMaxCTAs * 8);
    const size_t bytes = b_mom + b_u + 2 * b_x + 2 * b_a + b_p;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMalloc(&mu->base, bytes);
    if (e != cudaSuccess) {
        delete mu;
        return fail(DBUF_ENOMEM, std::string("dbuf_muon_create: cudaMalloc: ") + cudaGetErrorString(e));
    }
    char* p = mu->base;
    mu->mom = reinterpret_cast<float*>(p); p += b_mom;
    mu->u = reinterpret_cast<float*>(p); p += b_u;
    mu->x = reinterpret_cast<__nv_bfloat16*>(p); p += b_x;
    mu->y = reinterpret_cast<__nv_bfloat16*>(p); p += b_x;
    mu->a = reinterpret_cast<__nv_bfloat16*>(p); p += b_a;
    mu->b = reinterpret_cast<__nv_bfloat16*>(p); p += b_a;
    mu->partial = reinterpret_cast<double*>(p);
    e = cudaMemsetAsync(mu->mom, 0, (size_t)total * 4, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) {
        dbuf_muon_destroy(mu);
        return fail(DBUF_ECUDA, std::string("dbuf_muon_create: ") + cudaGetErrorString(e));
    }
    if (cublasCreate(&mu->h) != CUBLAS_STATUS_SUCCESS) {
        mu->h = nullptr;
        dbuf_muon_destroy(mu);
        return fail(DBUF_ECUDA, "dbuf_muon_create: cublasCreate failed");
    }
    *out = mu;
    return DBUF_OK;
}

// ns_steps quintic iterations on the bf16 iterate mu->x, a rows x cols
// row-major matrix; the result is left in mu->x.  Viewed column-major, the
// buffer holds X^T (cols x rows).  Wide X (rows <= cols) iterates on X itself:
// A = X X^T is (X^T)^T (X^T), and X' = aX + BX is X'^T = a X^T + X^T B^T.  Tall X
// iterates on Y = X^T, the buffer's own column-major matrix: A = Y Y^T,
// Y' = aY + BY.
static dbuf_status newton_schulz(dbuf_muon_s* mu, int64_t R, int64_t C, int32_t steps, cudaStream_t cs) {
    const bool wide = R <= C;
    const int s = (int)(wide ? R : C), l = (int)(wide ? C : R);
    const float one = 1.f, zero = 0.f, ca = kNsA, cb = kNsB, cc = kNsC;
    const size_t xbytes = (size_t)R * C * 2, abytes = (size_t)s * s * 2;
    CUBLAS_TRY(cublasSetStream(mu->h, cs), "newton_schulz");
    for (int it = 0; it < steps; ++it) {
        // A = Y Y^T (s x s), Y the wide iterate.
        if (wide)
            CUBLAS_TRY(cublasGemmEx(mu->h, CUBLAS_OP_T, CUBLAS_OP_N, s, s, l, &one, mu->x, CUDA_R_16BF, l, mu->x,
                                    CUDA_R_16BF, l, &zero, mu->a, CUDA_R_16BF, s, CUBLAS_COMPUTE_32F,
                                    CUBLAS_GEMM_DEFAULT),
                       "newton_schulz: X X^T");
        else
            CUBLAS_TRY(cublasGemmEx(mu->h, CUBLAS_OP_N, CUBLAS_OP_T, s, s, l, &one, mu->x, CUDA_R_16BF, s, mu->x,
                                    CUDA_R_16BF, s, &zero, mu->a, CUDA_R_16BF, s, CUBLAS_COMPUTE_32F,
                                    CUBLAS_GEMM_DEFAULT),
                       "newton_schulz: Y Y^T");
        // B = b A + c A A
        CUDA_TRY(cudaMemcpyAsync(mu->b, mu->a, abytes, cudaMemcpyDeviceToDevice, cs), "newton_schulz: copy");
        CUBLAS_TRY(cublasGemmEx(mu->h, CUBLAS_OP_N, CUBLAS_OP_N, s, s, s, &cc, mu->a, CUDA_R_16BF, s, mu->a,
                                CUDA_R_16BF, s, &cb, mu->b, CUDA_R_16BF, s, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT),
                   "newton_schulz: A A");
        // Y' = a Y + (B Y), into the other buffer
        CUDA_TRY(cudaMemcpyAsync(mu->y, mu->x, xbytes, cudaMemcpyDeviceToDevice, cs), "newton_schulz: copy");
        if (wide)
            CUBLAS_TRY(cublasGemmEx(mu->h, CUBLAS_OP_N, CUBLAS_OP_T, l, s, s, &one, mu->x, CUDA_R_16BF, l, mu->b,
                                    CUDA_R_16BF, s, &ca, mu->y, CUDA_R_16BF, l, CUBLAS_COMPUTE_32F,
                                    CUBLAS_GEMM_DEFAULT),
                       "newton_schulz: X^T B^T");
        else
            CUBLAS_TRY(cublasGemmEx(mu->h, CUBLAS_OP_N, CUBLAS_OP_N, s, l, s, &one, mu->b, CUDA_R_16BF, s, mu->x,
                                    CUDA_R_16BF, s, &ca, mu->y, CUDA_R_16BF, s, CUBLAS_COMPUTE_32F,
                                    CUBLAS_GEMM_DEFAULT),
                       "newton_schulz: B Y");
        std::swap(mu->x, mu->y);
    }
    return DBUF_OK;
}

static dbuf_status normalise(dbuf_muon_s* mu, const float* u, int64_t n, float eps, cudaStream_t cs) {
    const int g = muon_grid(n);
    muon_normalise_kernel<<<g, kMuonThreads, 0, cs>>>(u, n, mu->partial, g, eps, mu->x);
    CUDA_TRY(cudaGetLastError(), "dbuf_muon: normalise launch");
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_muon_orthogonalize(dbuf_muon_t* mu, const float* u, int64_t rows, int64_t cols,
                                               int32_t ns_steps, float eps, void* x_bf16, void* stream) {
    if (!mu || !u || !x_bf16) return fail(DBUF_EINVAL, "dbuf_muon_orthogonalize: NULL argument");
    if (rows < 2 || cols < 2 || ns_steps < 0 || rows * cols > mu->cap_rc ||
        std::min(rows, cols) * std::min(rows, cols) > mu->cap_ss)
        return fail(DBUF_EINVAL, "dbuf_muon_orthogonalize: shape outside the state's workspace");
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const int64_t n = rows * cols;
    const int g = muon_grid(n);
    muon_sumsq_kernel<<<g, kMuonThreads, 0, cs>>>(u, n, mu->partial);
    CUDA_TRY(cudaGetLastError(), "dbuf_muon_orthogonalize: launch");
    dbuf_status st = normalise(mu, u, n, eps, cs);
    if (st == DBUF_OK) st = newton_schulz(mu, rows, cols, ns_steps, cs);
    if (st != DBUF_OK) return st;
    CUDA_TRY(cudaMemcpyAsync(x_bf16, mu->x, (size_t)n * 2, cudaMemcpyDeviceToDevice, cs), "dbuf_muon_orthogonalize");
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_muon_step(dbuf_muon_t* mu, const dbuf_muon_hparams* hp, float grad_scale, void* stream) {
    if (!mu || !hp) return fail(DBUF_EINVAL, "dbuf_muon_step: NULL argument");
    if (hp->ns_steps < 1 || !(hp->momentum >= 0.f && hp->momentum < 1.f))
        return fail(DBUF_EINVAL, "dbuf_muon_step: need ns_steps >= 1 and momentum in [0, 1)");
    int dev = -1;
    CUDA_TRY(cudaGetDevice(&dev), "dbuf_muon_step");
    if (dev != mu->device) return fail(DBUF_EINVAL, "dbuf_muon_step: wrong current device");
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const float decay = (float)(1.0 - (double)hp->lr * (double)hp->weight_decay);
    for (size_t j = 0; j < mu->ids.size(); ++j) {
        const int64_t R = mu->rows[j], C = mu->cols[j], n = R * C;
        const int g = muon_grid(n);
        muon_momentum_kernel<<<g, kMuonThreads, 0, cs>>>(mu->grad[j], mu->mom + mu->mom_off[j], mu->u, n,
                                                         hp->momentum, grad_scale, hp->nesterov, mu->partial);
        CUDA_TRY(cudaGetLastError(), "dbuf_muon_step: momentum launch");
        dbuf_status st = normalise(mu, mu->u, n, hp->eps, cs);
        if (st == DBUF_OK) st = newton_schulz(mu, R, C, hp->ns_steps, cs);
        if (st != DBUF_OK) return st;
        const float lrs = (float)((double)hp->lr * std::sqrt(std::max(1.0, (double)R / (double)C)));
        muon_update_kernel<<<g, kMuonThreads, 0, cs>>>(mu->master[j], mu->param[j], mu->x, n, decay, lrs);
        CUDA_TRY(cudaGetLastError(), "dbuf_muon_step: update launch");
    }
    return DBUF_OK;
}

extern "C" dbuf_status dbuf_muon_momentum(const dbuf_muon_t* mu, int32_t i, float** ptr, int64_t* n) {
    if (!mu || !ptr || !n || i < 0 || i >= (int32_t)mu->ids.size())
        return fail(DBUF_EINVAL, "dbuf_muon_momentum: bad argument");
    *ptr = mu->mom + mu->mom_off[i];
    *n = mu->rows[i] * mu->cols[i];
    return DBUF_OK;
}
