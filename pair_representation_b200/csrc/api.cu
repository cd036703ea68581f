// api.cu - the C ABI declared in include/trimul.h: argument checks, workspace
// carve-up, TMA descriptors and the launch sequence of the three stages.
//
// Nothing here allocates device memory or synchronises, except
// trimul_device_status, whose contract is to synchronise.
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <utility>

#include "atomattn.h"
#include "kernels.h"
#include "trimul.h"

using namespace trimul;

namespace {

constexpr int kMaxN = 16384;
constexpr size_t kHeader = 256;  // DeviceStatus lives at the start of the workspace
constexpr int kMaxDevices = 64;

thread_local char g_detail[512];

void set_detail(const char *what, cudaError_t e) {
    snprintf(g_detail, sizeof g_detail, "%s: %s (%d)", what, cudaGetErrorString(e), (int)e);
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
// Row pitch (elements) of the channel-major a, b, x sections. bf16 rows start on
// 128-byte boundaries, so every row of a TMA box covers whole 32-byte sectors and
// 128-byte lines (a pitch of N rounded to 8 leaves half the rows 16 bytes off a
// sector when N is not a multiple of 16); fp32 rows on 32-byte boundaries.
size_t ld_of(int N, int dtype = TRIMUL_DTYPE_BF16) {
    return dtype == TRIMUL_DTYPE_F32 ? round_up((size_t)N, 8) : round_up((size_t)N, 64);
}
size_t elem_size(int dtype) { return dtype == TRIMUL_DTYPE_F32 ? 4 : 2; }
size_t section_bytes(int N, int dtype) {
    return round_up((size_t)kC * (size_t)N * ld_of(N, dtype) * elem_size(dtype), 256);
}

bool valid_dtype(int d) { return d == TRIMUL_DTYPE_F32 || d == TRIMUL_DTYPE_BF16; }

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

bool overlap(const void *p, size_t pn, const void *q, size_t qn) {
    if (!p || !q || !pn || !qn) return false;
    const uintptr_t a = (uintptr_t)p, b = (uintptr_t)q;
    return a < b + qn && b < a + pn;
}

// ---- per-device state ------------------------------------------------------

struct DevState {
    bool init = false;
    int sms = 0;
    int cc_major = 0, cc_minor = 0;
    cudaError_t tc_setup = cudaSuccess;
};

std::mutex g_mu;
DevState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int device_state(const DevState **out, bool need_tc) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_detail("cudaGetDevice", e);
        return TRIMUL_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return TRIMUL_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    DevState &d = g_dev[dev];
    if (!d.init) {
        if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) {
            set_detail("cudaDeviceGetAttribute", e);
            return TRIMUL_ERR_CUDA;
        }
        if (d.cc_major == 10 && d.cc_minor == 0) {
            if ((e = prologue_tc_setup()) == cudaSuccess && (e = contract_tc_setup()) == cudaSuccess &&
                (e = epilogue_tc_setup()) == cudaSuccess && (e = backward_setup()) == cudaSuccess &&
                (e = atomattn_tc_setup()) == cudaSuccess)
                e = contract_mx_setup();
            d.tc_setup = e;
        } else {
            d.tc_setup = cudaErrorNoKernelImageForDevice;
        }
        if (!g_encode) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
            if (e == cudaSuccess && q == cudaDriverEntryPointSuccess && fn)
                g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        d.init = true;
    }
    if (need_tc) {
        if (d.cc_major != 10 || d.cc_minor != 0) {
            snprintf(g_detail, sizeof g_detail, "bf16 path needs sm_100 (found sm_%d%d)", d.cc_major, d.cc_minor);
            return TRIMUL_ERR_UNSUPPORTED;
        }
        if (d.tc_setup != cudaSuccess) {
            set_detail("kernel attribute setup", d.tc_setup);
            return TRIMUL_ERR_CUDA;
        }
        if (!g_encode) {
            snprintf(g_detail, sizeof g_detail, "cuTensorMapEncodeTiled entry point unavailable");
            return TRIMUL_ERR_CUDA;
        }
    }
    *out = &d;
    return TRIMUL_OK;
}

// A pointer the kernels dereference must be device (or managed) memory.
int check_device_ptr(const void *p, const char *name) {
    if (!p) return TRIMUL_OK;
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        set_detail(name, e);
        return TRIMUL_ERR_INVALID_ARG;
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged) {
        snprintf(g_detail, sizeof g_detail, "%s is not device memory", name);
        return TRIMUL_ERR_INVALID_ARG;
    }
    return TRIMUL_OK;
}

// ---- argument checks (pure host logic, no CUDA calls) ------------------------

int check_params_core(const trimul_params *p);

int check_params(const trimul_params *p) {
    if (int rc = check_params_core(p)) return rc;
    if (!p->workspace || p->workspace_bytes < trimul_workspace_size_dtype(p->N, p->c_z, p->c_h, p->dtype))
        return TRIMUL_ERR_WORKSPACE;
    if (!aligned(p->workspace, 256)) return TRIMUL_ERR_MISALIGNED;
    return TRIMUL_OK;
}

// Everything check_params checks except the size of the workspace.
int check_params_core(const trimul_params *p) {
    if (!p) return TRIMUL_ERR_INVALID_ARG;
    if (p->N < 1 || p->N > kMaxN || p->c_z < 1 || p->c_h < 1) return TRIMUL_ERR_INVALID_ARG;
    if (p->c_z != kC || p->c_h != kC || !valid_dtype(p->dtype)) return TRIMUL_ERR_UNSUPPORTED;
    if (!(p->ln_eps > 0.f) || p->ln_eps > 1.f) return TRIMUL_ERR_INVALID_ARG;
    const void *req[] = {p->w_a, p->w_ag, p->w_b, p->w_bg, p->w_g, p->w_o};
    for (const void *w : req) {
        if (!w) return TRIMUL_ERR_INVALID_ARG;
        if (!aligned(w, 16)) return TRIMUL_ERR_MISALIGNED;
    }
    const size_t es = elem_size(p->dtype);
    const void *vec[] = {p->ln_in_w, p->ln_in_b, p->b_a, p->b_ag, p->b_b, p->b_bg,
                         p->b_g, p->ln_out_w, p->ln_out_b, p->b_o};
    for (const void *v : vec)
        if (v && !aligned(v, es)) return TRIMUL_ERR_MISALIGNED;
    return TRIMUL_OK;
}

// ---- shard stage calls: explicit buffers, a grid of rows x N cells or a subset of channels ----

size_t shard_ws_bytes(int N, int rows) { return kHeader + round_up((size_t)rows * ld_of(N) * 2, 256); }

int check_shard(const trimul_params *p, int rows) {
    if (int rc = check_params_core(p)) return rc;
    if (p->dtype != TRIMUL_DTYPE_BF16) return TRIMUL_ERR_UNSUPPORTED;
    if (rows < 1 || rows > p->N) return TRIMUL_ERR_INVALID_ARG;
    if (!p->workspace || p->workspace_bytes < shard_ws_bytes(p->N, rows)) return TRIMUL_ERR_WORKSPACE;
    if (!aligned(p->workspace, 256)) return TRIMUL_ERR_MISALIGNED;
    return TRIMUL_OK;
}

int check_buffers(std::initializer_list<std::pair<const void *, size_t>> in,
                  std::initializer_list<std::pair<const void *, size_t>> out, const trimul_params *p) {
    for (auto &b : in)
        if (b.first && !aligned(b.first, 16)) return TRIMUL_ERR_MISALIGNED;
    for (auto &o : out) {
        if (!o.first) return TRIMUL_ERR_INVALID_ARG;
        if (!aligned(o.first, 16)) return TRIMUL_ERR_MISALIGNED;
        if (overlap(o.first, o.second, p->workspace, p->workspace_bytes)) return TRIMUL_ERR_ALIAS;
        for (auto &b : in)
            if (overlap(o.first, o.second, b.first, b.second)) return TRIMUL_ERR_ALIAS;
        for (auto &q : out)
            if (&q != &o && overlap(o.first, o.second, q.first, q.second)) return TRIMUL_ERR_ALIAS;
    }
    return TRIMUL_OK;
}

size_t pair_bytes(const trimul_params *p) { return (size_t)p->N * p->N * kC * elem_size(p->dtype); }
size_t mask_bytes(const trimul_params *p) { return (size_t)p->N * p->N * elem_size(p->dtype); }

int check_z(const trimul_params *p, const void *z) {
    if (!z) return TRIMUL_ERR_INVALID_ARG;
    if (!aligned(z, 16)) return TRIMUL_ERR_MISALIGNED;
    if (overlap(z, pair_bytes(p), p->workspace, p->workspace_bytes)) return TRIMUL_ERR_ALIAS;
    return TRIMUL_OK;
}

int check_mask(const trimul_params *p, const void *mask) {
    if (!mask) return TRIMUL_OK;
    if (!aligned(mask, elem_size(p->dtype))) return TRIMUL_ERR_MISALIGNED;
    if (overlap(mask, mask_bytes(p), p->workspace, p->workspace_bytes)) return TRIMUL_ERR_ALIAS;
    return TRIMUL_OK;
}

int check_out(const trimul_params *p, const void *out, const void *z, const void *mask) {
    if (!out) return TRIMUL_ERR_INVALID_ARG;
    if (!aligned(out, 16)) return TRIMUL_ERR_MISALIGNED;
    const size_t n = pair_bytes(p);
    if (overlap(out, n, z, n) || overlap(out, n, mask, mask_bytes(p)) ||
        overlap(out, n, p->workspace, p->workspace_bytes))
        return TRIMUL_ERR_ALIAS;
    return TRIMUL_OK;
}

int check_direction(int d) { return (d == TRIMUL_OUTGOING || d == TRIMUL_INCOMING) ? TRIMUL_OK : TRIMUL_ERR_INVALID_ARG; }

int check_weights_on_device(const trimul_params *p) {
    const void *all[] = {p->w_a, p->w_ag, p->w_b, p->w_bg, p->w_g, p->w_o, p->ln_in_w, p->ln_in_b,
                         p->b_a, p->b_ag, p->b_b, p->b_bg, p->b_g, p->ln_out_w, p->ln_out_b, p->b_o,
                         p->workspace};
    for (const void *v : all) {
        int rc = check_device_ptr(v, "weight/workspace pointer");
        if (rc) return rc;
    }
    return TRIMUL_OK;
}

// ---- workspace views ----------------------------------------------------------

struct Views {
    DeviceStatus *status;
    uint8_t *a, *b, *x;
    size_t ld;
};

Views views_of(const trimul_params *p) {
    Views v;
    uint8_t *base = static_cast<uint8_t *>(p->workspace);
    const size_t sec = section_bytes(p->N, p->dtype);
    v.status = reinterpret_cast<DeviceStatus *>(base);
    v.a = base + kHeader;
    v.b = v.a + sec;
    v.x = v.b + sec;
    v.ld = ld_of(p->N, p->dtype);
    return v;
}

KernelCtl ctl_of(const trimul_params *p, const Views &v) {
    KernelCtl c;
    c.status = v.status;
    c.timeout_ns = (unsigned long long)(p->timeout_ms ? p->timeout_ms : 2000u) * 1000000ull;
    c.debug_flags = p->debug_flags;
    return c;
}

// ---- tensor maps ----------------------------------------------------------------

int encode(CUtensorMap *m, int rank, const void *base, const uint64_t *dims, const uint64_t *strides,
           const uint32_t *box, CUtensorMapSwizzle sw,
           CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    cuuint64_t gd[5], gs[4];
    cuuint32_t bd[5], es[5];
    for (int r = 0; r < rank; ++r) {
        gd[r] = dims[r];
        bd[r] = box[r];
        es[r] = 1;
        if (r < rank - 1) gs[r] = strides[r];
    }
    CUresult res = g_encode(m, dt, (cuuint32_t)rank, const_cast<void *>(base), gd, gs,
                            bd, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (res != CUDA_SUCCESS) {
        snprintf(g_detail, sizeof g_detail, "cuTensorMapEncodeTiled failed (%d), rank %d", (int)res, rank);
        return TRIMUL_ERR_CUDA;
    }
    return TRIMUL_OK;
}

// 128 x 128 weight [out][in], loaded as two 64-column halves with 128-byte swizzle.
int map_weight(CUtensorMap *m, const void *w) {
    const uint64_t dims[2] = {128, 128}, strides[1] = {128 * 2};
    const uint32_t box[2] = {64, 128};
    return encode(m, 2, w, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// z or out [rows][N][128] as (c, j, i): box of b0 channels x b1 cells of one row.
int map_pair(CUtensorMap *m, const void *t, int N, int rows, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw) {
    const uint64_t dims[3] = {128, (uint64_t)N, (uint64_t)rows};
    const uint64_t strides[2] = {128 * 2, (uint64_t)N * 128 * 2};
    const uint32_t box[3] = {b0, b1, 1};
    return encode(m, 3, t, dims, strides, box, sw);
}

// mask [rows][pitch] as (j, i): one row segment of 128 cells per box, zero past column N.
int map_mask(CUtensorMap *m, const void *t, int N, int rows, size_t pitch) {
    const uint64_t dims[2] = {(uint64_t)N, (uint64_t)rows}, strides[1] = {pitch * 2};
    const uint32_t box[2] = {128, 1};
    return encode(m, 2, t, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// a, b or x [channels][rows][ld] (N columns) as (col, row, c) with the given box and swizzle.
int map_cm(CUtensorMap *m, const void *t, int N, size_t ld, uint32_t b0, uint32_t b1, uint32_t b2,
           CUtensorMapSwizzle sw, int rows = 0, int channels = 128) {
    if (rows == 0) rows = N;
    const uint64_t dims[3] = {(uint64_t)N, (uint64_t)rows, (uint64_t)channels};
    const uint64_t strides[2] = {ld * 2, (uint64_t)rows * ld * 2};
    const uint32_t box[3] = {b0, b1, b2};
    return encode(m, 3, t, dims, strides, box, sw);
}

F32Layer f32_layer(const trimul_params *p, const void *mask, const Views &v) {
    F32Layer L;
    L.N = p->N;
    L.ld = v.ld;
    L.eps = p->ln_eps;
    L.mask = static_cast<const float *>(mask);
    L.ln_in_w = static_cast<const float *>(p->ln_in_w);
    L.ln_in_b = static_cast<const float *>(p->ln_in_b);
    L.ln_out_w = static_cast<const float *>(p->ln_out_w);
    L.ln_out_b = static_cast<const float *>(p->ln_out_b);
    L.w_a = static_cast<const float *>(p->w_a);
    L.w_ag = static_cast<const float *>(p->w_ag);
    L.w_b = static_cast<const float *>(p->w_b);
    L.w_bg = static_cast<const float *>(p->w_bg);
    L.w_g = static_cast<const float *>(p->w_g);
    L.w_o = static_cast<const float *>(p->w_o);
    L.b_a = static_cast<const float *>(p->b_a);
    L.b_ag = static_cast<const float *>(p->b_ag);
    L.b_b = static_cast<const float *>(p->b_b);
    L.b_bg = static_cast<const float *>(p->b_bg);
    L.b_g = static_cast<const float *>(p->b_g);
    L.b_o = static_cast<const float *>(p->b_o);
    L.a = reinterpret_cast<float *>(v.a);
    L.b = reinterpret_cast<float *>(v.b);
    L.x = reinterpret_cast<float *>(v.x);
    return L;
}

int cuda_rc(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return TRIMUL_OK;
    set_detail(what, e);
    return TRIMUL_ERR_CUDA;
}

// ---- stages ------------------------------------------------------------------------

// The bf16 prologue over a grid of rows x N cells: z [rows][N][128], mask [rows][N]
// or null, a and b written as [128][rows][ld]. mask_scratch holds rows * ld bf16
// for a mask whose rows lack a 16-byte pitch.
// The launch fields every prologue mode shares (the tiling is set by the caller).
PrologueArgs prologue_args(const trimul_params *p, bool has_mask, const KernelCtl &ctl, bool clear) {
    PrologueArgs a;
    memset(&a, 0, sizeof a);
    a.N = p->N;
    a.eps = p->ln_eps;
    a.has_mask = has_mask;
    a.ln_w = static_cast<const __nv_bfloat16 *>(p->ln_in_w);
    a.ln_b = static_cast<const __nv_bfloat16 *>(p->ln_in_b);
    a.b_a = static_cast<const __nv_bfloat16 *>(p->b_a);
    a.b_ag = static_cast<const __nv_bfloat16 *>(p->b_ag);
    a.b_b = static_cast<const __nv_bfloat16 *>(p->b_b);
    a.b_bg = static_cast<const __nv_bfloat16 *>(p->b_bg);
    a.clear_status = clear ? 1 : 0;
    a.ctl = ctl;
    return a;
}

int map_weights(PrologueMaps *m, const trimul_params *p) {
    const void *w[4] = {p->w_a, p->w_ag, p->w_b, p->w_bg};
    for (int k = 0; k < 4; ++k)
        if (int rc = map_weight(&m->w[k], w[k])) return rc;
    return TRIMUL_OK;
}

int clear_status(const trimul_params *p, cudaStream_t s);

// clear: this launch starts the call, so the kernel zeroes the status word (no separate
// memset in the stream).
int run_prologue_tc(const void *z, const void *mask, const trimul_params *p, int rows, void *a_out, void *b_out,
                    void *mask_scratch, const KernelCtl &ctl, const DevState &d, cudaStream_t s, bool clear) {
    const size_t ld = ld_of(p->N);
    PrologueMaps m;
    if (int rc = map_weights(&m, p)) return rc;
    if (int rc = map_pair(&m.z, z, p->N, rows, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return rc;
    // The mask rows travel with the z tiles. A tensor map needs a 16-byte row pitch, so a
    // mask whose rows do not have one is first copied into the scratch with pitch ld.
    m.mask = m.z;  // unused without a mask
    if (mask) {
        const void *src = mask;
        size_t pitch = (size_t)p->N;
        if (p->N % 8 != 0 || !aligned(mask, 16)) {
            __nv_bfloat16 *pad = reinterpret_cast<__nv_bfloat16 *>(mask_scratch);
            if (int rc = cuda_rc(launch_mask_pad(static_cast<const __nv_bfloat16 *>(mask), pad, p->N, rows, (int)ld, s),
                                 "mask_pad launch"))
                return rc;
            src = pad;
            pitch = ld;
        }
        if (int rc = map_mask(&m.mask, src, p->N, rows, pitch)) return rc;
    }
    // Each gating warp stores 32 cells x 32 channels (64-byte rows, 64-byte swizzle).
    if (int rc = map_cm(&m.a, a_out, p->N, ld, 32, 1, 32, CU_TENSOR_MAP_SWIZZLE_64B, rows)) return rc;
    if (int rc = map_cm(&m.b, b_out, p->N, ld, 32, 1, 32, CU_TENSOR_MAP_SWIZZLE_64B, rows)) return rc;
    PrologueArgs a = prologue_args(p, mask != nullptr, ctl, clear);
    a.jt_tiles = (p->N + 127) / 128;
    a.total_tiles = rows * a.jt_tiles;
    const int grid = a.total_tiles < d.sms ? a.total_tiles : d.sms;
    return cuda_rc(launch_prologue_tc(m, a, PRO_BF16, grid, s), "prologue_tc launch");
}

int run_prologue(const void *z, const void *mask, const trimul_params *p, const DevState &d, cudaStream_t s,
                 bool clear) {
    const Views v = views_of(p);
    if (p->dtype == TRIMUL_DTYPE_F32) {
        if (clear)
            if (int rc = clear_status(p, s)) return rc;
        const long tiles = (long)p->N * ((p->N + 31) / 32);
        const int grid = (int)(tiles < (long)d.sms * 8 ? tiles : (long)d.sms * 8);
        return cuda_rc(launch_prologue_f32(static_cast<const float *>(z), f32_layer(p, mask, v), grid, s),
                       "prologue_f32 launch");
    }
    // A re-pitched mask goes to plane 0 of x, which the contraction overwrites later.
    return run_prologue_tc(z, mask, p, p->N, v.a, v.b, v.x, ctl_of(p, v), d, s, clear);
}

// A matrix operand of the pair kernel: element (row, col) of batch b at
// ptr + b * batch_stride + row * row_stride + col (elements).
struct MatView {
    const void *ptr;
    size_t row_stride, batch_stride;
};

// 3-D (col, row, batch) tensor map over a MatView with `cols` x `rows` elements.
int map_view(CUtensorMap *m, const MatView &v, int cols, int rows, int batch, uint32_t b0, uint32_t b1, int es,
             CUtensorMapDataType dt) {
    const uint64_t dims[3] = {(uint64_t)cols, (uint64_t)rows, (uint64_t)batch};
    // A single matrix still needs a valid (non-zero, 16-byte multiple) batch stride.
    const size_t bs = batch > 1 ? v.batch_stride : v.row_stride * (size_t)rows;
    const uint64_t strides[2] = {v.row_stride * es, bs * es};
    const uint32_t box[3] = {b0, b1, 1};
    return encode(m, 3, v.ptr, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, dt);
}

// X_b[m][n] = sum_k A_b(m, k) B_b(n, k) on the tcgen05 pair kernel for m < M,
// n < Ncols, k < K and every batch index b; A and B bf16, each K-major
// ([rows][k]: row = m or n) or MN-major ([k][rows]); X bf16 or fp32. CTA pairs
// share each 256 x 256 output tile: CTA r loads rows [128 r, 128 r + 128) of the
// A and B panels (boxes of 128 rows, or 2 x 64-wide blocks when MN-major).
int run_gemm(const MatView &A, int a_mn, const MatView &B, int b_mn, const MatView &X, int out_f32, int M, int Ncols,
             int K, int batch, const KernelCtl &ctl, const DevState &d, cudaStream_t s) {
    ContractMaps m;
    const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (int rc = a_mn ? map_view(&m.a, A, M, K, batch, 64, 64, 2, bf) : map_view(&m.a, A, K, M, batch, 64, 128, 2, bf))
        return rc;
    if (int rc = b_mn ? map_view(&m.b, B, Ncols, K, batch, 64, 64, 2, bf)
                      : map_view(&m.b, B, K, Ncols, batch, 64, 128, 2, bf))
        return rc;
    // X is stored by each drain warp in blocks of 32 rows x 128 bytes.
    if (int rc = out_f32 ? map_view(&m.x, X, Ncols, M, batch, 32, 32, 4, CU_TENSOR_MAP_DATA_TYPE_FLOAT32)
                         : map_view(&m.x, X, Ncols, M, batch, 64, 32, 2, bf))
        return rc;
    ContractArgs a;
    a.M = M;
    a.Ncols = Ncols;
    a.K = K;
    a.a_mn = a_mn;
    a.b_mn = b_mn;
    a.ti_tiles = (M + 255) / 256;
    a.tj_tiles = (Ncols + 255) / 256;
    a.total_tiles = batch * a.ti_tiles * a.tj_tiles;
    a.kblocks = (K + 63) / 64;
    a.out_f32 = out_f32;
    a.ctl = ctl;
    const int pairs = a.total_tiles < d.sms / 2 ? a.total_tiles : d.sms / 2;
    return cuda_rc(launch_contract_tc(m, a, 2 * pairs, s), "contract_tc launch");
}

// The triangle contraction X_c = A_c B_c^T in general form over `channels`
// channel-major [channels][N][ld] bf16 arrays, each operand K-major ([rows][k])
// or MN-major ([k][rows]).
int run_contract_on(const void *A, int a_mn, const void *B, int b_mn, void *X, int N, size_t ld, const KernelCtl &ctl,
                    const DevState &d, cudaStream_t s, int channels = kC) {
    const size_t cs = (size_t)N * ld;
    return run_gemm({A, ld, cs}, a_mn, {B, ld, cs}, b_mn, {X, ld, cs}, 0, N, N, N, channels, ctl, d, s);
}

int run_contract(const trimul_params *p, int direction, const DevState &d, cudaStream_t s) {
    const Views v = views_of(p);
    if (p->dtype == TRIMUL_DTYPE_F32)
        return cuda_rc(launch_contract_f32(f32_layer(p, nullptr, v), direction, s), "contract_f32 launch");
    const int mn = direction == TRIMUL_INCOMING;
    return run_contract_on(v.a, mn, v.b, mn, v.x, p->N, v.ld, ctl_of(p, v), d, s);
}

// The bf16 epilogue over a grid of rows x N cells: z and out [rows][N][128], x [128][rows][ld].
int run_epilogue_tc(const void *z, const void *x, const trimul_params *p, int rows, void *out, const KernelCtl &ctl,
                    const DevState &d, cudaStream_t s) {
    EpilogueMaps m;
    if (int rc = map_weight(&m.wg, p->w_g)) return rc;
    if (int rc = map_weight(&m.wo, p->w_o)) return rc;
    if (int rc = map_pair(&m.z, z, p->N, rows, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return rc;
    // x as the MN-major MMA operand: 64 cells x 128 channels per box, 128-byte swizzle.
    if (int rc = map_cm(&m.x, x, p->N, ld_of(p->N), 64, 1, 128, CU_TENSOR_MAP_SWIZZLE_128B, rows)) return rc;
    // Each worker warp stores 32 channels x 32 cells (64-byte rows, 64-byte swizzle).
    if (int rc = map_pair(&m.out, out, p->N, rows, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)) return rc;
    EpilogueArgs a;
    a.N = p->N;
    a.jt_tiles = (p->N + 127) / 128;
    a.total_tiles = rows * a.jt_tiles;
    a.eps = p->ln_eps;
    a.ln_in_w = static_cast<const __nv_bfloat16 *>(p->ln_in_w);
    a.ln_in_b = static_cast<const __nv_bfloat16 *>(p->ln_in_b);
    a.ln_out_w = static_cast<const __nv_bfloat16 *>(p->ln_out_w);
    a.ln_out_b = static_cast<const __nv_bfloat16 *>(p->ln_out_b);
    a.b_g = static_cast<const __nv_bfloat16 *>(p->b_g);
    a.b_o = static_cast<const __nv_bfloat16 *>(p->b_o);
    a.ctl = ctl;
    const int grid = a.total_tiles < d.sms ? a.total_tiles : d.sms;
    return cuda_rc(launch_epilogue_tc(m, a, grid, s), "epilogue_tc launch");
}

int run_epilogue(const void *z, const trimul_params *p, void *out, const DevState &d, cudaStream_t s) {
    const Views v = views_of(p);
    if (p->dtype == TRIMUL_DTYPE_F32) {
        const long tiles = (long)p->N * ((p->N + 31) / 32);
        const int grid = (int)(tiles < (long)d.sms * 8 ? tiles : (long)d.sms * 8);
        return cuda_rc(launch_epilogue_f32(static_cast<const float *>(z), static_cast<float *>(out),
                                           f32_layer(p, nullptr, v), grid, s),
                       "epilogue_f32 launch");
    }
    return run_epilogue_tc(z, v.x, p, p->N, out, ctl_of(p, v), d, s);
}

int clear_status(const trimul_params *p, cudaStream_t s) {
    return cuda_rc(cudaMemsetAsync(p->workspace, 0, sizeof(DeviceStatus), s), "status clear");
}

// ---- MXFP8 contraction -----------------------------------------------------------------

// Sections after the bf16 workspace (each 256-byte aligned): the E4M3 operands
// aq, bq [128][N][ldq] and their scales sa (per 128-row half of a 256-row pair
// tile), sb (per 192-row tile), both per 128-wide K chunk.
struct MxLayout {
    size_t aq, bq, sa, sb, total, ldq;
    int ti, tj, kc;
};

MxLayout mx_layout(int N) {
    MxLayout L;
    L.ldq = ((size_t)N + 15) & ~(size_t)15;
    L.ti = (N + 255) / 256;
    L.tj = (N + 191) / 192;
    L.kc = (N + 127) / 128;
    size_t off = kHeader + 3 * section_bytes(N, TRIMUL_DTYPE_BF16);
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = round_up(off + bytes, 256);
        return o;
    };
    L.aq = take((size_t)kC * N * L.ldq);
    L.bq = take((size_t)kC * N * L.ldq);
    L.sa = take((size_t)kC * 2 * L.ti * L.kc * 512);
    L.sb = take((size_t)kC * L.tj * L.kc * 1024);
    L.total = off;
    return L;
}

int check_mx(const trimul_params *p) {
    if (p->dtype != TRIMUL_DTYPE_BF16) return TRIMUL_ERR_UNSUPPORTED;
    if (p->workspace_bytes < mx_layout(p->N).total) return TRIMUL_ERR_WORKSPACE;
    return TRIMUL_OK;
}

int run_contract_mx_mma(const trimul_params *p, const DevState &d, cudaStream_t s);

int run_contract_mx(const trimul_params *p, int direction, const DevState &d, cudaStream_t s) {
    const Views v = views_of(p);
    const int N = p->N;
    const MxLayout L = mx_layout(N);
    uint8_t *base = static_cast<uint8_t *>(p->workspace);
    const int tr = direction == TRIMUL_INCOMING;  // incoming: operand row m is the column of a and b
    // The last 192-row tile of b has scale slots no row reaches; they must not hold NaN codes.
    if (int rc = cuda_rc(cudaMemsetAsync(base + L.sb, 0, (size_t)kC * L.tj * L.kc * 1024, s), "mx scale clear"))
        return rc;
    MxQuantArgs q;
    q.N = N;
    q.ld = v.ld;
    q.ldq = L.ldq;
    q.kchunks = L.kc;
    q.src = reinterpret_cast<const __nv_bfloat16 *>(v.a);
    q.q = base + L.aq;
    q.sf = base + L.sa;
    q.rows_per_tile = 128;
    q.row_tiles = 2 * L.ti;
    q.chunks_per_tile = 1;
    if (int rc = cuda_rc(launch_mx_quant(q, tr, s), "mx_quant launch")) return rc;
    q.src = reinterpret_cast<const __nv_bfloat16 *>(v.b);
    q.q = base + L.bq;
    q.sf = base + L.sb;
    q.rows_per_tile = 192;
    q.row_tiles = L.tj;
    q.chunks_per_tile = 2;
    if (int rc = cuda_rc(launch_mx_quant(q, tr, s), "mx_quant launch")) return rc;
    return run_contract_mx_mma(p, d, s);
}

// The block-scaled contraction of the MXFP8 operands already in the workspace into x.
int run_contract_mx_mma(const trimul_params *p, const DevState &d, cudaStream_t s) {
    const Views v = views_of(p);
    const int N = p->N;
    const MxLayout L = mx_layout(N);
    uint8_t *base = static_cast<uint8_t *>(p->workspace);
    ContractMxMaps m;
    const uint64_t qdims[3] = {(uint64_t)N, (uint64_t)N, (uint64_t)kC};
    const uint64_t qstr[2] = {L.ldq, (uint64_t)N * L.ldq};
    const uint32_t abox[3] = {128, 128, 1}, bbox[3] = {128, 96, 1};
    if (int rc = encode(&m.a, 3, base + L.aq, qdims, qstr, abox, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_DATA_TYPE_UINT8))
        return rc;
    if (int rc = encode(&m.b, 3, base + L.bq, qdims, qstr, bbox, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_DATA_TYPE_UINT8))
        return rc;
    const uint64_t sadims[2] = {16, (uint64_t)kC * 2 * L.ti * L.kc * 32}, sbdims[2] = {16, (uint64_t)kC * L.tj * L.kc * 64};
    const uint64_t sstr[1] = {16};
    const uint32_t sabox[2] = {16, 32}, sbbox[2] = {16, 64};
    if (int rc = encode(&m.sa, 2, base + L.sa, sadims, sstr, sabox, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_DATA_TYPE_UINT8))
        return rc;
    if (int rc = encode(&m.sb, 2, base + L.sb, sbdims, sstr, sbbox, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_DATA_TYPE_UINT8))
        return rc;
    if (int rc = map_cm(&m.x, v.x, N, v.ld, 64, 32, 1, CU_TENSOR_MAP_SWIZZLE_128B)) return rc;
    ContractMxArgs a;
    a.N = N;
    a.ti_tiles = L.ti;
    a.tj_tiles = L.tj;
    a.total_tiles = kC * L.ti * L.tj;
    a.kchunks = L.kc;
    a.a_row_tiles = 2 * L.ti;
    a.b_row_tiles = L.tj;
    a.ctl = ctl_of(p, v);
    const int pairs = a.total_tiles < d.sms / 2 ? a.total_tiles : d.sms / 2;
    return cuda_rc(launch_contract_mx(m, a, 2 * pairs, s), "contract_mx launch");
}

// The prologue writing the MXFP8 operands of `direction`'s contraction (E4M3 codes
// and scales) straight into the MX sections of the workspace: outgoing on row
// tiles, incoming on 32 x 4 column tiles (the contracted index of a_ki is the row).
int run_prologue_mx(const void *z, const void *mask, const trimul_params *p, int direction, const DevState &d,
                    cudaStream_t s, bool clear) {
    const Views v = views_of(p);
    const int N = p->N;
    const MxLayout L = mx_layout(N);
    uint8_t *base = static_cast<uint8_t *>(p->workspace);
    const bool cols = direction == TRIMUL_INCOMING;
    // The contraction reads whole 128-wide K chunks: the scales of K blocks past the last
    // residue (zero codes, no cell writes them) must be finite, so both arrays start at 0.
    if (int rc = cuda_rc(cudaMemsetAsync(base + L.sa, 0, (size_t)kC * 2 * L.ti * L.kc * 512, s), "mx scale clear"))
        return rc;
    if (int rc = cuda_rc(cudaMemsetAsync(base + L.sb, 0, (size_t)kC * L.tj * L.kc * 1024, s), "mx scale clear"))
        return rc;
    PrologueMaps m;
    if (int rc = map_weights(&m, p)) return rc;
    if (cols) {
        // (c, j, i) over z, one column's 32 rows per box.
        const uint64_t dims[3] = {128, (uint64_t)N, (uint64_t)N};
        const uint64_t strides[2] = {128 * 2, (uint64_t)N * 128 * 2};
        const uint32_t box[3] = {64, 1, 32};
        if (int rc = encode(&m.z, 3, z, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return rc;
    } else if (int rc = map_pair(&m.z, z, N, N, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) {
        return rc;
    }
    m.mask = m.z;  // unused without a mask
    if (mask) {
        // Re-pitched (row tiles) or transposed (column tiles) into plane 0 of x, which
        // the contraction overwrites later.
        __nv_bfloat16 *scratch = reinterpret_cast<__nv_bfloat16 *>(v.x);
        const __nv_bfloat16 *mk = static_cast<const __nv_bfloat16 *>(mask);
        if (cols) {
            if (int rc = cuda_rc(launch_mask_transpose(mk, scratch, N, (int)v.ld, s), "mask_transpose launch"))
                return rc;
            const uint64_t dims[2] = {(uint64_t)N, (uint64_t)N}, strides[1] = {(uint64_t)v.ld * 2};
            const uint32_t box[2] = {32, 4};
            if (int rc = encode(&m.mask, 2, scratch, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE)) return rc;
        } else {
            const void *src = mask;
            size_t pitch = (size_t)N;
            if (N % 8 != 0 || !aligned(mask, 16)) {
                if (int rc = cuda_rc(launch_mask_pad(mk, scratch, N, N, (int)v.ld, s), "mask_pad launch")) return rc;
                src = scratch;
                pitch = v.ld;
            }
            if (int rc = map_mask(&m.mask, src, N, N, pitch)) return rc;
        }
    }
    // E4M3 operands [c][N][ldq] as (k, row, c); each gating warp stores 32 channels x 32 bytes.
    const uint64_t qdims[3] = {(uint64_t)N, (uint64_t)N, (uint64_t)kC};
    const uint64_t qstr[2] = {L.ldq, (uint64_t)N * L.ldq};
    const uint32_t qbox[3] = {32, 1, 32};
    if (int rc = encode(&m.a, 3, base + L.aq, qdims, qstr, qbox, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_DATA_TYPE_UINT8))
        return rc;
    if (int rc = encode(&m.b, 3, base + L.bq, qdims, qstr, qbox, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_DATA_TYPE_UINT8))
        return rc;
    PrologueArgs a = prologue_args(p, mask != nullptr, ctl_of(p, v), clear);
    if (cols) {
        a.jt_tiles = (N + 3) / 4;
        a.total_tiles = ((N + 31) / 32) * a.jt_tiles;
    } else {
        a.jt_tiles = (N + 127) / 128;
        a.total_tiles = N * a.jt_tiles;
    }
    a.sf[0] = base + L.sa;
    a.sf[1] = base + L.sb;
    a.sf_rows[0] = 128;
    a.sf_row_tiles[0] = 2 * L.ti;
    a.sf_chunks[0] = 1;
    a.sf_rows[1] = 192;
    a.sf_row_tiles[1] = L.tj;
    a.sf_chunks[1] = 2;
    a.kchunks = L.kc;
    const int grid = a.total_tiles < d.sms ? a.total_tiles : d.sms;
    return cuda_rc(launch_prologue_tc(m, a, cols ? PRO_MX_COLS : PRO_MX_ROWS, grid, s), "prologue_tc launch");
}

// ---- backward ----------------------------------------------------------------------

constexpr long long kWgradChunk = 4096;  // cells per weight-gradient GEMM partial

// Weight-gradient partials of one block of R rows: one per kWgradChunk cells.
long long wgrad_slots(int N, int R) { return ((long long)R * N + kWgradChunk - 1) / kWgradChunk; }

// Sections of the backward workspace (byte offsets, each 256-byte aligned) for
// blocks of R rows: the per-cell intermediates and the weight-gradient partials
// hold one block (R N cells); dX, dA, dB (channel-major) and dP_G (only when
// R < N) cover the whole grid.
struct BwdLayout {
    size_t sums, wstack, wacc, st_in, st_out, zh, xh, P, Y, dxh, D, dy, dg, dX, dA, dB, partial, total;
};

BwdLayout bwd_layout(int N, int R) {
    const size_t M = (size_t)R * N, C = kC, cm = C * (size_t)N * ld_of(N);
    BwdLayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = round_up(off + bytes, 256);
        return o;
    };
    L.sums = take((size_t)kSumCount * C * 4);
    L.wstack = take((size_t)kProjBlocks * C * C * 2);
    L.wacc = take((size_t)kWgradRows * C * 8);   // weight-gradient sums over the blocks, double
    L.st_in = take(M * 8);
    L.st_out = take(M * 8);
    L.zh = take(M * C * 2);                 // LayerNorm_in(z), bf16 [cells][128]
    L.xh = take(M * C * 2);                 // LayerNorm_out(x), bf16 [cells][128]
    L.P = take(M * kProjBlocks * C * 2);    // zh W^T pre-activations, bf16; later dL/dzh, fp32 [cells][128]
    L.Y = take(M * C * 2);                  // xh W_o^T, bf16
    L.dxh = take(M * C * 4);                // dL/dxh, fp32
    L.D = take(M * kProjBlocks * C * 2);    // pre-activation gradients, bf16
    L.dy = take(M * C * 2);                 // dL/dy, bf16
    L.dg = R < N ? take((size_t)N * N * C * 2) : 0;  // dP_G of every cell, bf16 [cells][128]
    L.dX = take(cm * 2);                    // dL/dx, bf16 [128][N][ld]
    L.dA = take(cm * 2);                    // dL/da, bf16 [128][N][ld]
    L.dB = take(cm * 2);
    L.partial = take((size_t)wgrad_slots(N, R) * kWgradRows * C * 4);
    L.total = off;
    return L;
}

// The largest block of rows whose layout fits `bytes` (0 if none does). Below N
// the size grows with the rows; the whole grid (R = N) needs no dP_G copy, so
// it is tried first and can fit where N - 1 rows do not.
int bwd_rows_for(int N, size_t bytes) {
    if (bwd_layout(N, N).total <= bytes) return N;
    if (N == 1 || bwd_layout(N, 1).total > bytes) return 0;
    int lo = 1, hi = N - 1;  // fits(lo); find the largest fitting R in [lo, hi]
    if (bwd_layout(N, hi).total <= bytes) return hi;
    while (hi - lo > 1) {  // fits(lo), !fits(hi)
        const int mid = lo + (hi - lo) / 2;
        (bwd_layout(N, mid).total <= bytes ? lo : hi) = mid;
    }
    return lo;
}

int check_backward(const trimul_params *p, const void *z, const void *mask, const void *dout, const void *dz,
                   const trimul_grads *g) {
    if (!dout || !dz || !g) return TRIMUL_ERR_INVALID_ARG;
    if (p->dtype != TRIMUL_DTYPE_BF16) return TRIMUL_ERR_UNSUPPORTED;
    if (!aligned(dout, 16) || !aligned(dz, 16)) return TRIMUL_ERR_MISALIGNED;
    if (!g->workspace || bwd_rows_for(p->N, g->workspace_bytes) < 1) return TRIMUL_ERR_WORKSPACE;
    if (!aligned(g->workspace, 256)) return TRIMUL_ERR_MISALIGNED;
    const size_t n = pair_bytes(p), mb = mask_bytes(p);
    const void *gws = g->workspace;
    const size_t gwn = g->workspace_bytes;
    if (overlap(dz, n, z, n) || overlap(dz, n, mask, mb) || overlap(dz, n, dout, n) ||
        overlap(dz, n, p->workspace, p->workspace_bytes) || overlap(dz, n, gws, gwn) ||
        overlap(dout, n, p->workspace, p->workspace_bytes) || overlap(dout, n, gws, gwn) ||
        overlap(gws, gwn, p->workspace, p->workspace_bytes) || overlap(gws, gwn, z, n) || overlap(gws, gwn, mask, mb))
        return TRIMUL_ERR_ALIAS;
    // Gradient outputs: weights [128][128] (16-byte aligned, written by GEMMs), vectors [128].
    const void *outs[16] = {g->d_w_a, g->d_w_ag, g->d_w_b, g->d_w_bg, g->d_w_g, g->d_w_o,
                            g->d_b_a, g->d_b_ag, g->d_b_b, g->d_b_bg, g->d_b_g, g->d_b_o,
                            g->d_ln_in_w, g->d_ln_in_b, g->d_ln_out_w, g->d_ln_out_b};
    size_t sz[16];
    for (int k = 0; k < 16; ++k) {
        sz[k] = (size_t)(k < 6 ? kC * kC : kC) * 4;
        if (outs[k] && !aligned(outs[k], k < 6 ? 16 : 4)) return TRIMUL_ERR_MISALIGNED;
    }
    for (int k = 0; k < 16; ++k) {
        if (!outs[k]) continue;
        if (overlap(outs[k], sz[k], z, n) || overlap(outs[k], sz[k], mask, mb) || overlap(outs[k], sz[k], dout, n) ||
            overlap(outs[k], sz[k], dz, n) || overlap(outs[k], sz[k], p->workspace, p->workspace_bytes) ||
            overlap(outs[k], sz[k], gws, gwn))
            return TRIMUL_ERR_ALIAS;
        for (int l = k + 1; l < 16; ++l)
            if (overlap(outs[k], sz[k], outs[l], sz[l])) return TRIMUL_ERR_ALIAS;
    }
    return TRIMUL_OK;
}

int check_backward_on_device(const void *dout, const void *dz, const trimul_grads *g) {
    const void *all[] = {dout, dz, g->workspace, g->d_w_a, g->d_w_ag, g->d_w_b, g->d_w_bg, g->d_w_g, g->d_w_o,
                         g->d_b_a, g->d_b_ag, g->d_b_b, g->d_b_bg, g->d_b_g, g->d_b_o,
                         g->d_ln_in_w, g->d_ln_in_b, g->d_ln_out_w, g->d_ln_out_b};
    for (const void *v : all)
        if (int rc = check_device_ptr(v, "backward pointer")) return rc;
    return TRIMUL_OK;
}

// The backward's launch sequence. The per-cell steps run over blocks of R rows
// (R = N when the workspace holds the whole grid, else as many rows as fit): a
// first pass per block down to dL/dx, the contraction's adjoint over the whole
// grid, then a second pass per block down to dL/dz. With R < N the second pass
// recomputes zh and the a/b pre-activations of its block, and takes dP_G from
// the whole-grid copy the first pass left; with R = N it reuses the first
// pass's zh and P. The arithmetic of every cell is the same either way.
int run_backward(const void *z, const void *mask, const trimul_params *p, int direction, const void *dout, void *dz,
                 const trimul_grads *gr, const DevState &d, cudaStream_t s) {
    typedef __nv_bfloat16 bf;
    const int N = p->N, C = kC, PB = kProjBlocks * kC;
    const int R = bwd_rows_for(N, gr->workspace_bytes);
    const bool blocked = R < N;
    const Views v = views_of(p);
    const BwdLayout L = bwd_layout(N, R);
    uint8_t *base = static_cast<uint8_t *>(gr->workspace);
    float *sums = reinterpret_cast<float *>(base + L.sums);
    bf *wstack = reinterpret_cast<bf *>(base + L.wstack);
    float2 *st_in = reinterpret_cast<float2 *>(base + L.st_in), *st_out = reinterpret_cast<float2 *>(base + L.st_out);
    bf *zh = reinterpret_cast<bf *>(base + L.zh), *xh = reinterpret_cast<bf *>(base + L.xh);
    bf *P = reinterpret_cast<bf *>(base + L.P), *Y = reinterpret_cast<bf *>(base + L.Y);
    float *dzh = reinterpret_cast<float *>(base + L.P), *dxh = reinterpret_cast<float *>(base + L.dxh);
    bf *D = reinterpret_cast<bf *>(base + L.D), *dy = reinterpret_cast<bf *>(base + L.dy);
    bf *dg_all = blocked ? reinterpret_cast<bf *>(base + L.dg) : nullptr;
    bf *dX = reinterpret_cast<bf *>(base + L.dX);
    bf *dA = reinterpret_cast<bf *>(base + L.dA), *dB = reinterpret_cast<bf *>(base + L.dB);
    float *partial = reinterpret_cast<float *>(base + L.partial);
    double *wacc = reinterpret_cast<double *>(base + L.wacc);
    const bf *x = reinterpret_cast<const bf *>(v.x);
    const bf *zb = static_cast<const bf *>(z), *doutb = static_cast<const bf *>(dout);
    bf *dzb = static_cast<bf *>(dz);
    int rc;

    // Recompute the forward's a, b and x into the forward workspace, unless the caller
    // states that the last forward call left them there.
    if ((rc = clear_status(p, s))) return rc;
    if (!(gr->flags & TRIMUL_BWD_REUSE_FORWARD) &&
        ((rc = run_prologue(z, mask, p, d, s, false)) || (rc = run_contract(p, direction, d, s))))
        return rc;
    if ((rc = cuda_rc(cudaMemsetAsync(sums, 0, (size_t)kSumCount * C * 4, s), "backward sums clear"))) return rc;
    const void *wk[kProjBlocks] = {p->w_g, p->w_a, p->w_ag, p->w_b, p->w_bg};
    for (int k = 0; k < kProjBlocks; ++k)
        if ((rc = cuda_rc(cudaMemcpyAsync(wstack + (size_t)k * C * C, wk[k], (size_t)C * C * 2,
                                          cudaMemcpyDeviceToDevice, s), "weight stack copy")))
            return rc;

    // The plain GEMMs run on the pair kernel (run_gemm): X[m][n] = sum_k A(m, k) B(n, k),
    // each operand K-major or MN-major (mn = 1), bf16 in, fp32 accumulation.
    const KernelCtl ctl = ctl_of(p, v);
    const size_t ck = (size_t)kWgradChunk, pstride = (size_t)kWgradRows * C;
    float *wdst[kProjBlocks + 1] = {gr->d_w_g, gr->d_w_a, gr->d_w_ag, gr->d_w_b, gr->d_w_bg, gr->d_w_o};
    // Weight gradients of one block: for each kWgradChunk cells of it, rows row0 ..
    // row0 + arows of one partial get the sum over the chunk's cells of A[cell][r]
    // Bm[cell][c] (both operands MN-major: the contracted index is the cell, their row
    // index; the chunks are the GEMM's batch); then the partials are added, in
    // double, to the sums over the blocks, which the last block writes out.
    auto wgrad = [&](const bf *A, int arows, size_t lda, const bf *Bm, long long ncells, int row0, bool first,
                     bool last) -> int {
        const long long full = ncells / kWgradChunk, rem = ncells - full * kWgradChunk;
        float *dst = partial + (size_t)row0 * C;
        int r;
        if (full > 0 && (r = run_gemm({A, lda, ck * lda}, 1, {Bm, (size_t)C, ck * C}, 1, {dst, (size_t)C, pstride}, 1,
                                      arows, C, (int)kWgradChunk, (int)full, ctl, d, s)))
            return r;
        if (rem > 0 && (r = run_gemm({A + (size_t)full * ck * lda, lda, ck * lda}, 1, {Bm + (size_t)full * ck * C,
                                      (size_t)C, ck * C}, 1, {dst + (size_t)full * pstride, (size_t)C, pstride}, 1,
                                      arows, C, (int)rem, 1, ctl, d, s)))
            return r;
        WgradReduceArgs wr;
        wr.partial = partial;
        wr.slots = (int)(full + (rem > 0));
        wr.row0 = row0;
        wr.rows = arows;
        wr.acc = wacc;
        wr.first = first;
        wr.last = last;
        for (int k = 0; k <= kProjBlocks; ++k) wr.dst[k] = wdst[k];
        return cuda_rc(launch_wgrad_reduce(wr, s), "wgrad_reduce launch");
    };

    LnFwdArgs lf;
    lf.N = N;
    lf.ld = v.ld;
    lf.eps = p->ln_eps;
    LnBwdArgs lb;
    lb.N = N;
    lb.ld = v.ld;
    // LayerNorm_in of the block's z rows into zh (and its statistics).
    auto ln_in = [&](int r0, int nr) {
        lf.src = zb + (size_t)r0 * N * C;
        lf.channel_major = 0;
        lf.rows = nr;
        lf.i0 = r0;
        lf.gamma = static_cast<const bf *>(p->ln_in_w);
        lf.beta = static_cast<const bf *>(p->ln_in_b);
        lf.out = zh;
        lf.stats = st_in;
        return cuda_rc(launch_ln_fwd(lf, d.sms, s), "ln_fwd launch");
    };

    // ---- first pass, per block of rows: down to dL/dx ----
    for (int r0 = 0; r0 < N; r0 += R) {
        const int nr = N - r0 < R ? N - r0 : R, M = nr * N;
        if ((rc = ln_in(r0, nr))) return rc;
        lf.src = x;
        lf.channel_major = 1;
        lf.gamma = static_cast<const bf *>(p->ln_out_w);
        lf.beta = static_cast<const bf *>(p->ln_out_b);
        lf.out = xh;
        lf.stats = st_out;
        if ((rc = cuda_rc(launch_ln_fwd(lf, d.sms, s), "ln_fwd launch"))) return rc;
        // P = zh [W_g; W_a; W_ag; W_b; W_bg]^T (only its P_G block when the second pass
        // recomputes the rest) and Y = xh W_o^T, before biases, bf16.
        if ((rc = run_gemm({zh, (size_t)C, 0}, 0, {wstack, (size_t)C, 0}, 0, {P, (size_t)PB, 0}, 0, M,
                           blocked ? C : PB, C, 1, ctl, d, s)) ||
            (rc = run_gemm({xh, (size_t)C, 0}, 0, {p->w_o, (size_t)C, 0}, 0, {Y, (size_t)C, 0}, 0, M, C, C, 1, ctl, d,
                           s)))
            return rc;

        GateBwdArgs ga;
        ga.dout = doutb + (size_t)r0 * N * C;
        ga.P = P;
        ga.Y = Y;
        ga.b_g = static_cast<const bf *>(p->b_g);
        ga.b_o = static_cast<const bf *>(p->b_o);
        ga.dy = dy;
        ga.dg = blocked ? dg_all + (size_t)r0 * N * C : D + P_G * C;
        ga.dg_stride = blocked ? (size_t)C : (size_t)PB;
        ga.db_g = sums + S_B_G * C;
        ga.db_o = sums + S_B_O * C;
        ga.cells = M;
        if ((rc = cuda_rc(launch_gate_bwd(ga, d.sms, s), "gate_bwd launch"))) return rc;

        // dL/dxh = dy W_o (fp32): B(n, k) = W_o[k][n] is MN-major.
        if ((rc = run_gemm({dy, (size_t)C, 0}, 0, {p->w_o, (size_t)C, 0}, 1, {dxh, (size_t)C, 0}, 1, M, C, C, 1, ctl,
                           d, s)))
            return rc;

        lb.dh = dxh;
        lb.src = x;
        lb.channel_major = 1;
        lb.rows = nr;
        lb.i0 = r0;
        lb.stats = st_out;
        lb.gamma = static_cast<const bf *>(p->ln_out_w);
        lb.dsrc = dX;
        lb.dgamma = sums + S_LN_OUT_W * C;
        lb.dbeta = sums + S_LN_OUT_B * C;
        if ((rc = cuda_rc(launch_ln_bwd(lb, d.sms, s), "ln_bwd launch"))) return rc;
        // W_o gradient partials: dy^T xh.
        if ((rc = wgrad(dy, C, (size_t)C, xh, M, PB, r0 == 0, r0 + nr == N))) return rc;
    }

    // The contraction's adjoint on the forward's contraction kernel, in the
    // form X[m][n] = sum_k A(m, k) B(n, k) with each operand K- or MN-major:
    //   outgoing (x_ij = sum_k a_ik b_jk):
    //     dA[i][k] = sum_j dX[i][j] b[j][k]   A = dX (K-major), B = b (MN-major)
    //     dB[j][k] = sum_i dX[i][j] a[i][k]   A = dX (MN-major), B = a (MN-major)
    //   incoming (x_ij = sum_k a_ki b_kj):
    //     dA[k][i] = sum_j b[k][j] dX[i][j]   A = b (K-major), B = dX (K-major)
    //     dB[k][j] = sum_i a[k][i] dX[i][j]   A = a (K-major), B = dX (MN-major)
    if (direction == TRIMUL_OUTGOING) {
        if ((rc = run_contract_on(dX, 0, v.b, 1, dA, N, v.ld, ctl, d, s)) ||
            (rc = run_contract_on(dX, 1, v.a, 1, dB, N, v.ld, ctl, d, s)))
            return rc;
    } else {
        if ((rc = run_contract_on(v.b, 0, dX, 0, dA, N, v.ld, ctl, d, s)) ||
            (rc = run_contract_on(v.a, 0, dX, 1, dB, N, v.ld, ctl, d, s)))
            return rc;
    }

    // ---- second pass, per block of rows: down to dL/dz ----
    for (int r0 = 0; r0 < N; r0 += R) {
        const int nr = N - r0 < R ? N - r0 : R, M = nr * N;
        if (blocked) {
            // zh and P_A .. P_BG of the block again; its dP_G into D's first block.
            if ((rc = ln_in(r0, nr)) ||
                (rc = run_gemm({zh, (size_t)C, 0}, 0, {wstack + (size_t)C * C, (size_t)C, 0}, 0, {P + C, (size_t)PB, 0},
                               0, M, PB - C, C, 1, ctl, d, s)) ||
                (rc = cuda_rc(cudaMemcpy2DAsync(D, (size_t)PB * 2, dg_all + (size_t)r0 * N * C, (size_t)C * 2,
                                                (size_t)C * 2, (size_t)M, cudaMemcpyDeviceToDevice, s),
                              "dP_G copy")))
                return rc;
        }

        ProjBwdArgs pa;
        pa.dA = dA;
        pa.dB = dB;
        pa.P = P;
        pa.mask = static_cast<const bf *>(mask);
        pa.b_a = static_cast<const bf *>(p->b_a);
        pa.b_ag = static_cast<const bf *>(p->b_ag);
        pa.b_b = static_cast<const bf *>(p->b_b);
        pa.b_bg = static_cast<const bf *>(p->b_bg);
        pa.D = D;
        pa.db = sums + S_B_A * C;
        pa.N = N;
        pa.rows = nr;
        pa.i0 = r0;
        pa.ld = v.ld;
        if ((rc = cuda_rc(launch_proj_bwd(pa, d.sms, s), "proj_bwd launch"))) return rc;

        // [W_g; W_a; W_ag; W_b; W_bg] gradient partials: D^T zh.
        if ((rc = wgrad(D, PB, (size_t)PB, zh, M, 0, r0 == 0, r0 + nr == N))) return rc;

        // dL/dzh = D [W_g; W_a; W_ag; W_b; W_bg] (fp32, over the spent pre-activations):
        // B(n, k) = Wstack[k][n] is MN-major.
        if ((rc = run_gemm({D, (size_t)PB, 0}, 0, {wstack, (size_t)C, 0}, 1, {dzh, (size_t)C, 0}, 1, M, C, PB, 1, ctl,
                           d, s)))
            return rc;

        lb.dh = dzh;
        lb.src = zb + (size_t)r0 * N * C;
        lb.channel_major = 0;
        lb.rows = nr;
        lb.i0 = r0;
        lb.stats = st_in;
        lb.gamma = static_cast<const bf *>(p->ln_in_w);
        lb.dsrc = dzb + (size_t)r0 * N * C;
        lb.dgamma = sums + S_LN_IN_W * C;
        lb.dbeta = sums + S_LN_IN_B * C;
        if ((rc = cuda_rc(launch_ln_bwd(lb, d.sms, s), "ln_bwd launch"))) return rc;
    }

    float *vec[kSumCount] = {gr->d_b_g, gr->d_b_o, gr->d_b_a, gr->d_b_ag, gr->d_b_b, gr->d_b_bg,
                             gr->d_ln_out_w, gr->d_ln_out_b, gr->d_ln_in_w, gr->d_ln_in_b};
    for (int k = 0; k < kSumCount; ++k)
        if (vec[k] && (rc = cuda_rc(cudaMemcpyAsync(vec[k], sums + k * C, (size_t)C * 4, cudaMemcpyDeviceToDevice, s),
                                    "gradient copy")))
            return rc;
    return TRIMUL_OK;
}

// ---- atom attention ------------------------------------------------------------------

size_t attn_elems(const atomattn_params *p) { return (size_t)p->batch * p->n_atoms * p->heads * 32; }
int attn_windows(const atomattn_params *p) { return (p->n_atoms + 31) / 32; }

int check_attn(const atomattn_params *p, const void *out) {
    if (!p || !out || !p->q || !p->k || !p->v) return TRIMUL_ERR_INVALID_ARG;
    if (p->batch < 1 || p->n_atoms < 1 || p->heads < 1) return TRIMUL_ERR_INVALID_ARG;
    if (p->batch > (1 << 20) || p->n_atoms > (1 << 26)) return TRIMUL_ERR_INVALID_ARG;
    if (p->head_dim != 32 || p->heads > 64) return TRIMUL_ERR_UNSUPPORTED;
    if ((long long)p->batch * p->heads * ((p->n_atoms + 127) / 128) > 0x7fffffffLL) return TRIMUL_ERR_UNSUPPORTED;
    const void *al16[] = {p->q, p->k, p->v, p->bias, out};
    for (const void *v : al16)
        if (v && !aligned(v, 16)) return TRIMUL_ERR_MISALIGNED;
    if (p->atom_mask && !aligned(p->atom_mask, 2)) return TRIMUL_ERR_MISALIGNED;
    if (!p->workspace || p->workspace_bytes < atomattn_workspace_size()) return TRIMUL_ERR_WORKSPACE;
    if (!aligned(p->workspace, 256)) return TRIMUL_ERR_MISALIGNED;
    const size_t n = attn_elems(p) * 2;
    const size_t nb = (size_t)p->batch * attn_windows(p) * p->heads * 32 * 128 * 2;
    const size_t nm = (size_t)p->batch * p->n_atoms * 2;
    if (overlap(out, n, p->q, n) || overlap(out, n, p->k, n) || overlap(out, n, p->v, n) ||
        overlap(out, n, p->bias, nb) || overlap(out, n, p->atom_mask, nm) ||
        overlap(out, n, p->workspace, p->workspace_bytes))
        return TRIMUL_ERR_ALIAS;
    return TRIMUL_OK;
}

// q, k or v [batch][n][heads][32] as (heads * 32, n, batch): boxes of one head's 32 elements x `rows`.
int map_attn(CUtensorMap *m, const void *t, const atomattn_params *p, uint32_t rows) {
    const uint64_t row = (uint64_t)p->heads * 32;
    const uint64_t dims[3] = {row, (uint64_t)p->n_atoms, (uint64_t)p->batch};
    const uint64_t strides[2] = {row * 2, row * 2 * (uint64_t)p->n_atoms};
    const uint32_t box[3] = {32, rows, 1};
    return encode(m, 3, t, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B);
}

// bias [batch][n_windows][heads][32][128] as (slot, row, head, window, batch): boxes of one
// window's 32 rows x 64 slots; windows past n_windows read as 0.
int map_attn_bias(CUtensorMap *m, const atomattn_params *p) {
    const uint64_t nw = (uint64_t)attn_windows(p), h = (uint64_t)p->heads;
    const uint64_t dims[5] = {128, 32, h, nw, (uint64_t)p->batch};
    const uint64_t strides[4] = {128 * 2, 32 * 128 * 2, h * 32 * 128 * 2, nw * h * 32 * 128 * 2};
    const uint32_t box[5] = {64, 32, 1, 1, 1};
    return encode(m, 5, p->bias, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

// ---- exported symbols -------------------------------------------------------------

extern "C" {

size_t trimul_workspace_size_dtype(int N, int c_z, int c_h, int dtype) {
    if (N < 1 || N > kMaxN || c_z != kC || c_h != kC || !valid_dtype(dtype)) return 0;
    return kHeader + 3 * section_bytes(N, dtype);
}

size_t trimul_workspace_size(int N, int c_z, int c_h) {
    return trimul_workspace_size_dtype(N, c_z, c_h, TRIMUL_DTYPE_F32);
}

int trimul_prologue(const void *z, const void *mask, const trimul_params *p, trimul_stream_t stream) {
    int rc;
    if ((rc = check_params(p)) || (rc = check_z(p, z)) || (rc = check_mask(p, mask))) return rc;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, p->dtype == TRIMUL_DTYPE_BF16))) return rc;
    if ((rc = check_weights_on_device(p)) || (rc = check_device_ptr(z, "z")) ||
        (rc = check_device_ptr(mask, "mask")))
        return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return run_prologue(z, mask, p, *d, s, true);
}

int trimul_contract(const trimul_params *p, int direction, trimul_stream_t stream) {
    int rc;
    if ((rc = check_params(p)) || (rc = check_direction(direction))) return rc;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, p->dtype == TRIMUL_DTYPE_BF16))) return rc;
    if ((rc = check_device_ptr(p->workspace, "workspace"))) return rc;
    return run_contract(p, direction, *d, reinterpret_cast<cudaStream_t>(stream));
}

int trimul_epilogue(const void *z, const trimul_params *p, void *out, trimul_stream_t stream) {
    int rc;
    if ((rc = check_params(p)) || (rc = check_z(p, z)) || (rc = check_out(p, out, z, nullptr))) return rc;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, p->dtype == TRIMUL_DTYPE_BF16))) return rc;
    if ((rc = check_weights_on_device(p)) || (rc = check_device_ptr(z, "z")) || (rc = check_device_ptr(out, "out")))
        return rc;
    return run_epilogue(z, p, out, *d, reinterpret_cast<cudaStream_t>(stream));
}

int trimul_forward(const void *z, const void *mask, const trimul_params *p, int direction, void *out,
                   trimul_stream_t stream) {
    int rc;
    if ((rc = check_params(p)) || (rc = check_direction(direction)) || (rc = check_z(p, z)) ||
        (rc = check_mask(p, mask)) || (rc = check_out(p, out, z, mask)))
        return rc;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, p->dtype == TRIMUL_DTYPE_BF16))) return rc;
    if ((rc = check_weights_on_device(p)) || (rc = check_device_ptr(z, "z")) ||
        (rc = check_device_ptr(mask, "mask")) || (rc = check_device_ptr(out, "out")))
        return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = run_prologue(z, mask, p, *d, s, true))) return rc;
    if ((rc = run_contract(p, direction, *d, s))) return rc;
    return run_epilogue(z, p, out, *d, s);
}

size_t trimul_workspace_size_mxfp8(int N, int c_z, int c_h) {
    if (N < 1 || N > kMaxN || c_z != kC || c_h != kC) return 0;
    return mx_layout(N).total;
}

int trimul_contract_mxfp8(const trimul_params *p, int direction, trimul_stream_t stream) {
    int rc;
    if ((rc = check_params(p)) || (rc = check_direction(direction)) || (rc = check_mx(p))) return rc;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, true))) return rc;
    if ((rc = check_device_ptr(p->workspace, "workspace"))) return rc;
    return run_contract_mx(p, direction, *d, reinterpret_cast<cudaStream_t>(stream));
}

int trimul_forward_mxfp8(const void *z, const void *mask, const trimul_params *p, int direction, void *out,
                         trimul_stream_t stream) {
    int rc;
    if ((rc = check_params(p)) || (rc = check_direction(direction)) || (rc = check_mx(p)) || (rc = check_z(p, z)) ||
        (rc = check_mask(p, mask)) || (rc = check_out(p, out, z, mask)))
        return rc;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, true))) return rc;
    if ((rc = check_weights_on_device(p)) || (rc = check_device_ptr(z, "z")) ||
        (rc = check_device_ptr(mask, "mask")) || (rc = check_device_ptr(out, "out")))
        return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = run_prologue_mx(z, mask, p, direction, *d, s, true))) return rc;
    if ((rc = run_contract_mx_mma(p, *d, s))) return rc;
    return run_epilogue(z, p, out, *d, s);
}

int trimul_prologue_mxfp8(const void *z, const void *mask, const trimul_params *p, int direction,
                          trimul_stream_t stream) {
    int rc;
    if ((rc = check_params(p)) || (rc = check_direction(direction)) || (rc = check_mx(p)) || (rc = check_z(p, z)) ||
        (rc = check_mask(p, mask)))
        return rc;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, true))) return rc;
    if ((rc = check_weights_on_device(p)) || (rc = check_device_ptr(z, "z")) ||
        (rc = check_device_ptr(mask, "mask")) || (rc = check_device_ptr(p->workspace, "workspace")))
        return rc;
    return run_prologue_mx(z, mask, p, direction, *d, reinterpret_cast<cudaStream_t>(stream), false);
}

int trimul_mma_mxfp8(const trimul_params *p, trimul_stream_t stream) {
    int rc;
    if ((rc = check_params(p)) || (rc = check_mx(p))) return rc;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, true))) return rc;
    if ((rc = check_device_ptr(p->workspace, "workspace"))) return rc;
    return run_contract_mx_mma(p, *d, reinterpret_cast<cudaStream_t>(stream));
}

int trimul_mxfp8_views(const trimul_params *p, void **aq, void **bq, void **sa, void **sb, size_t *ldq) {
    int rc;
    if ((rc = check_params(p)) || (rc = check_mx(p))) return rc;
    const MxLayout L = mx_layout(p->N);
    uint8_t *base = static_cast<uint8_t *>(p->workspace);
    if (aq) *aq = base + L.aq;
    if (bq) *bq = base + L.bq;
    if (sa) *sa = base + L.sa;
    if (sb) *sb = base + L.sb;
    if (ldq) *ldq = L.ldq;
    return TRIMUL_OK;
}

size_t trimul_shard_workspace_size(int N, int rows) {
    if (N < 1 || N > kMaxN || rows < 1 || rows > N) return 0;
    return shard_ws_bytes(N, rows);
}

int trimul_prologue_rows(const void *z_rows, const void *mask_rows, const trimul_params *p, int rows, void *a,
                         void *b, trimul_stream_t stream) {
    int rc;
    if ((rc = check_shard(p, rows))) return rc;
    if (!z_rows) return TRIMUL_ERR_INVALID_ARG;
    const size_t nz = (size_t)rows * p->N * kC * 2, nm = (size_t)rows * p->N * 2;
    const size_t nab = (size_t)kC * rows * ld_of(p->N) * 2;
    if ((rc = check_buffers({{z_rows, nz}}, {{a, nab}, {b, nab}}, p))) return rc;
    // The mask needs only element alignment: rows without a 16-byte pitch are re-pitched.
    if (mask_rows && !aligned(mask_rows, 2)) return TRIMUL_ERR_MISALIGNED;
    if (overlap(a, nab, mask_rows, nm) || overlap(b, nab, mask_rows, nm) ||
        overlap(mask_rows, nm, p->workspace, p->workspace_bytes))
        return TRIMUL_ERR_ALIAS;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, true))) return rc;
    const void *dev[] = {z_rows, mask_rows, a, b};
    for (const void *v : dev)
        if ((rc = check_device_ptr(v, "shard buffer"))) return rc;
    if ((rc = check_weights_on_device(p))) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Views v = views_of(p);
    return run_prologue_tc(z_rows, mask_rows, p, rows, a, b, static_cast<uint8_t *>(p->workspace) + kHeader,
                           ctl_of(p, v), *d, s, true);
}

int trimul_contract_channels(const trimul_params *p, int direction, int channels, const void *a, const void *b,
                             void *x, trimul_stream_t stream) {
    int rc;
    if ((rc = check_shard(p, 1)) || (rc = check_direction(direction))) return rc;
    if (channels < 1 || channels > kC || !a || !b) return TRIMUL_ERR_INVALID_ARG;
    const size_t n = (size_t)channels * p->N * ld_of(p->N) * 2;
    if ((rc = check_buffers({{a, n}, {b, n}}, {{x, n}}, p))) return rc;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, true))) return rc;
    const void *dev[] = {a, b, x, p->workspace};
    for (const void *v : dev)
        if ((rc = check_device_ptr(v, "shard buffer"))) return rc;
    const int mn = direction == TRIMUL_INCOMING;
    const Views v = views_of(p);
    return run_contract_on(a, mn, b, mn, x, p->N, ld_of(p->N), ctl_of(p, v), *d,
                           reinterpret_cast<cudaStream_t>(stream), channels);
}

int trimul_epilogue_rows(const void *z_rows, const void *x_rows, const trimul_params *p, int rows, void *out_rows,
                         trimul_stream_t stream) {
    int rc;
    if ((rc = check_shard(p, rows))) return rc;
    if (!z_rows || !x_rows) return TRIMUL_ERR_INVALID_ARG;
    const size_t nz = (size_t)rows * p->N * kC * 2, nx = (size_t)kC * rows * ld_of(p->N) * 2;
    if ((rc = check_buffers({{z_rows, nz}, {x_rows, nx}}, {{out_rows, nz}}, p))) return rc;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, true))) return rc;
    const void *dev[] = {z_rows, x_rows, out_rows};
    for (const void *v : dev)
        if ((rc = check_device_ptr(v, "shard buffer"))) return rc;
    if ((rc = check_weights_on_device(p))) return rc;
    const Views v = views_of(p);
    return run_epilogue_tc(z_rows, x_rows, p, rows, out_rows, ctl_of(p, v), *d, reinterpret_cast<cudaStream_t>(stream));
}

int trimul_workspace_views(const trimul_params *p, void **a, void **b, void **x, size_t *ld) {
    int rc = check_params(p);
    if (rc) return rc;
    const Views v = views_of(p);
    if (a) *a = v.a;
    if (b) *b = v.b;
    if (x) *x = v.x;
    if (ld) *ld = v.ld;
    return TRIMUL_OK;
}

int trimul_device_status(const trimul_params *p, trimul_stream_t stream, int *detail) {
    if (!p) return TRIMUL_ERR_INVALID_ARG;
    // Without a workspace the status word is the one in the static scratch of
    // trimul_forward_noalloc on the current device.
    const void *word = p->workspace;
    if (!word) {
        void *scratch = nullptr;
        if (int rc = noalloc_scratch_address(&scratch)) return rc;
        word = scratch;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DeviceStatus st;
    cudaError_t e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemcpy(&st, word, sizeof st, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
        set_detail("status read", e);
        return TRIMUL_ERR_CUDA;
    }
    if (detail) {
        detail[0] = st.code;
        detail[1] = st.site;
        detail[2] = st.block;
        detail[3] = st.aux;
    }
    if (st.code == DEV_OK) return TRIMUL_OK;
    return st.code == DEV_TIMEOUT ? TRIMUL_ERR_TIMEOUT : TRIMUL_ERR_DEVICE;
}

size_t trimul_backward_workspace_size(int N, int c_z, int c_h) {
    if (N < 1 || N > kMaxN || c_z != kC || c_h != kC) return 0;
    return bwd_layout(N, N).total;
}

size_t trimul_backward_workspace_size_rows(int N, int c_z, int c_h, int rows) {
    if (N < 1 || N > kMaxN || c_z != kC || c_h != kC || rows < 1 || rows > N) return 0;
    return bwd_layout(N, rows).total;
}

int trimul_backward_block_rows(int N, int c_z, int c_h, size_t workspace_bytes) {
    if (N < 1 || N > kMaxN || c_z != kC || c_h != kC) return 0;
    return bwd_rows_for(N, workspace_bytes);
}

int trimul_backward(const void *z, const void *mask, const trimul_params *p, int direction, const void *dout,
                    void *dz, const trimul_grads *g, trimul_stream_t stream) {
    int rc;
    if ((rc = check_params(p)) || (rc = check_direction(direction)) || (rc = check_z(p, z)) ||
        (rc = check_mask(p, mask)) || (rc = check_backward(p, z, mask, dout, dz, g)))
        return rc;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, true))) return rc;
    if ((rc = check_weights_on_device(p)) || (rc = check_device_ptr(z, "z")) ||
        (rc = check_device_ptr(mask, "mask")) || (rc = check_backward_on_device(dout, dz, g)))
        return rc;
    return run_backward(z, mask, p, direction, dout, dz, g, *d, reinterpret_cast<cudaStream_t>(stream));
}

size_t atomattn_workspace_size(void) { return kHeader; }

int atomattn_forward(const atomattn_params *p, void *out, trimul_stream_t stream) {
    int rc;
    if ((rc = check_attn(p, out))) return rc;
    const DevState *d = nullptr;
    if ((rc = device_state(&d, true))) return rc;
    const void *ptrs[] = {p->q, p->k, p->v, p->bias, p->atom_mask, p->workspace, out};
    for (const void *v : ptrs)
        if ((rc = check_device_ptr(v, "atom attention pointer"))) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // The kernel clears the status word itself (CTA 0, after its setup barrier).
    AttnMaps m;
    if ((rc = map_attn(&m.q, p->q, p, 128)) || (rc = map_attn(&m.k, p->k, p, 224)) ||
        (rc = map_attn(&m.v, p->v, p, 256)))
        return rc;
    m.bias = m.q;  // unused without a bias
    if (p->bias && (rc = map_attn_bias(&m.bias, p))) return rc;
    AttnArgs a;
    a.batch = p->batch;
    a.n = p->n_atoms;
    a.heads = p->heads;
    a.groups = (p->n_atoms + 127) / 128;
    a.n_windows = attn_windows(p);
    a.units = (long long)p->batch * p->heads * a.groups;
    a.bias = static_cast<const __nv_bfloat16 *>(p->bias);
    a.mask = static_cast<const __nv_bfloat16 *>(p->atom_mask);
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.scale = 0.17677669529663687f;  // 1 / sqrt(32)
    a.ctl.status = static_cast<DeviceStatus *>(p->workspace);
    a.ctl.timeout_ns = (unsigned long long)(p->timeout_ms ? p->timeout_ms : 2000u) * 1000000ull;
    a.ctl.debug_flags = 0;
    const int grid = a.units < d->sms ? (int)a.units : d->sms;
    return cuda_rc(launch_atomattn_tc(m, a, grid, s), "atomattn_tc launch");
}

int atomattn_device_status(const atomattn_params *p, trimul_stream_t stream, int *detail) {
    if (!p || !p->workspace) return TRIMUL_ERR_INVALID_ARG;
    DeviceStatus st;
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = cudaMemcpy(&st, p->workspace, sizeof st, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
        set_detail("status read", e);
        return TRIMUL_ERR_CUDA;
    }
    if (detail) {
        detail[0] = st.code;
        detail[1] = st.site;
        detail[2] = st.block;
        detail[3] = st.aux;
    }
    if (st.code == DEV_OK) return TRIMUL_OK;
    return st.code == DEV_TIMEOUT ? TRIMUL_ERR_TIMEOUT : TRIMUL_ERR_DEVICE;
}

const char *trimul_error_string(int code) {
    switch (code) {
        case TRIMUL_OK: return "ok";
        case TRIMUL_ERR_INVALID_ARG: return "invalid argument";
        case TRIMUL_ERR_UNSUPPORTED: return "unsupported configuration";
        case TRIMUL_ERR_MISALIGNED: return "pointer not aligned";
        case TRIMUL_ERR_ALIAS: return "output overlaps an input or the workspace";
        case TRIMUL_ERR_WORKSPACE: return "workspace missing or too small";
        case TRIMUL_ERR_CUDA: return "CUDA runtime or driver error";
        case TRIMUL_ERR_TIMEOUT: return "a bounded in-kernel wait ran out";
        case TRIMUL_ERR_DEVICE: return "kernel-detected fault";
        default: return "unknown status";
    }
}

const char *trimul_last_error_detail(void) { return g_detail; }

int trimul_version(void) { return 100; }

}  // extern "C"
