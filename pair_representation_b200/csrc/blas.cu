// blas.cu - cuBLAS for the backward's plain GEMMs, loaded with dlopen on first
// use so that the forward library has no link-time dependency on it.
//
// Row-major C[M][N] = op(A) op(B) is the column-major product
// C^T = op(B)^T op(A)^T, so each call hands cuBLAS the operands swapped, with
// (N, M, K); a transposed row-major operand becomes CUBLAS_OP_T.
#include <cublas_v2.h>
#include <dlfcn.h>

#include <cstdio>
#include <mutex>

#include "kernels.h"

namespace trimul {
namespace {

struct BlasApi {
    bool tried = false;
    void *lib = nullptr;
    decltype(&cublasCreate_v2) create = nullptr;
    decltype(&cublasSetStream_v2) set_stream = nullptr;
    decltype(&cublasSetWorkspace_v2) set_workspace = nullptr;
    // The header overloads this name in C++, so spell out the C entry point's type.
    cublasStatus_t (*gemm_sb)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int, const void *,
                              const void *, cudaDataType, int, long long, const void *, cudaDataType, int, long long,
                              const void *, void *, cudaDataType, int, long long, int, cublasComputeType_t,
                              cublasGemmAlgo_t) = nullptr;
};

constexpr int kMaxDev = 64;
std::mutex g_blas_mu;  // guards g_api and g_handle
std::mutex g_use_mu;   // blas_lock(): held by a caller across one sequence of GEMMs
BlasApi g_api;
cublasHandle_t g_handle[kMaxDev] = {};

bool load_api(char *detail, size_t n) {
    if (g_api.tried) {
        if (!g_api.gemm_sb) snprintf(detail, n, "cuBLAS unavailable (libcublas.so.12 not loaded)");
        return g_api.gemm_sb != nullptr;
    }
    g_api.tried = true;
    const char *names[] = {"libcublas.so.12", "/usr/local/cuda/lib64/libcublas.so.12"};
    for (const char *nm : names)
        if ((g_api.lib = dlopen(nm, RTLD_NOW | RTLD_LOCAL))) break;
    if (!g_api.lib) {
        snprintf(detail, n, "dlopen libcublas.so.12 failed: %s", dlerror());
        return false;
    }
    g_api.create = reinterpret_cast<decltype(g_api.create)>(dlsym(g_api.lib, "cublasCreate_v2"));
    g_api.set_stream = reinterpret_cast<decltype(g_api.set_stream)>(dlsym(g_api.lib, "cublasSetStream_v2"));
    g_api.set_workspace = reinterpret_cast<decltype(g_api.set_workspace)>(dlsym(g_api.lib, "cublasSetWorkspace_v2"));
    g_api.gemm_sb = reinterpret_cast<decltype(g_api.gemm_sb)>(dlsym(g_api.lib, "cublasGemmStridedBatchedEx"));
    if (!g_api.create || !g_api.set_stream || !g_api.set_workspace || !g_api.gemm_sb) {
        g_api.gemm_sb = nullptr;
        snprintf(detail, n, "libcublas.so.12 lacks an entry point");
        return false;
    }
    return true;
}

}  // namespace

void blas_lock() { g_use_mu.lock(); }
void blas_unlock() { g_use_mu.unlock(); }

int blas_bind(cudaStream_t s, void *ws, size_t ws_bytes, void **handle, char *detail, size_t n) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        snprintf(detail, n, "no current CUDA device");
        return -1;
    }
    std::lock_guard<std::mutex> lk(g_blas_mu);
    if (!load_api(detail, n)) return -1;
    if (!g_handle[dev]) {
        cublasStatus_t st = g_api.create(&g_handle[dev]);
        if (st != CUBLAS_STATUS_SUCCESS) {
            g_handle[dev] = nullptr;
            snprintf(detail, n, "cublasCreate failed (%d)", (int)st);
            return -1;
        }
    }
    // Setting the stream resets the workspace to cuBLAS's own pool, so bind both.
    cublasStatus_t st = g_api.set_stream(g_handle[dev], s);
    if (st == CUBLAS_STATUS_SUCCESS) st = g_api.set_workspace(g_handle[dev], ws, ws_bytes);
    if (st != CUBLAS_STATUS_SUCCESS) {
        snprintf(detail, n, "cublasSetStream/SetWorkspace failed (%d)", (int)st);
        return -1;
    }
    *handle = g_handle[dev];
    return 0;
}

int blas_gemm(void *handle, const Gemm &g, char *detail, size_t n) {
    const float one = 1.f;
    const cublasOperation_t opa = g.ta ? CUBLAS_OP_T : CUBLAS_OP_N;
    const cublasOperation_t opb = g.tb ? CUBLAS_OP_T : CUBLAS_OP_N;
    cublasStatus_t st = g_api.gemm_sb(static_cast<cublasHandle_t>(handle), opb, opa, g.N, g.M, g.K, &one, g.B,
                                      CUDA_R_16BF, g.ldb, g.sB, g.A, CUDA_R_16BF, g.lda, g.sA, &g.beta, g.C,
                                      g.c_f32 ? CUDA_R_32F : CUDA_R_16BF, g.ldc, g.sC, g.batch, CUBLAS_COMPUTE_32F,
                                      CUBLAS_GEMM_DEFAULT);
    if (st != CUBLAS_STATUS_SUCCESS) {
        snprintf(detail, n, "cublasGemmStridedBatchedEx failed (%d): M %d N %d K %d batch %d", (int)st, g.M, g.N, g.K,
                 g.batch);
        return (int)st;
    }
    return 0;
}

}  // namespace trimul
