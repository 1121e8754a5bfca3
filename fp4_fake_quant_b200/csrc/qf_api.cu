// qf_api.cu -- the C ABI of libqf.so (declared in include/qf.h): host-side argument
// validation, descriptor tables and kernel launches.  No memory is allocated; all
// work is enqueued on the caller's stream.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include "qf.h"
#include "qf_device.cuh"
#include "qf_lora.cuh"

#ifndef QF_LORA_STEP_TWO_PASS
#define QF_LORA_STEP_TWO_PASS 0  // LoRA step up to rank 16: 1 = pruned amax + fused NVFP4 pass
#endif
#include "qf_oneshot.cuh"

namespace {

using qf::DevTensor;
using qf::Table;
using qf::kThreads;

constexpr int kSmallT = 8;      // descriptor table sizes (kernel-parameter bytes: ~0.6 KB / ~27 KB)
constexpr int kLargeT = 384;
constexpr int kFp4U = QF_FP4_U;  // 256-element sub-tiles per warp unit
#ifndef QF_AMAX_U
#define QF_AMAX_U 4
#endif
constexpr int kAmaxU = QF_AMAX_U;
#ifndef QF_NV_REVERSE
#define QF_NV_REVERSE 1         // NVFP4 fused pass: units from the last one down (k_nv)
#endif
#ifndef QF_NOALLOC_MAX_GROUPS
#define QF_NOALLOC_MAX_GROUPS 4092     // 4 header words + 4092 slots = 16 KB of static scratch
#endif

thread_local char g_err[512] = "";

qf_status fail(qf_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return s;
}

qf_status cuda_fail(cudaError_t e, const char* what) {
    return fail(QF_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int block_of(qf_format f) { return f == QF_NVFP4 ? 16 : f == QF_MXFP4 ? 32 : 256; }

// Whether the byte ranges [a, a + na) and [b, b + nb) intersect (NULL or empty: no).
bool overlap(const void* a, int64_t na, const void* b, int64_t nb) {
    if (!a || !b || na <= 0 || nb <= 0) return false;
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + (uintptr_t)nb && pb < pa + (uintptr_t)na;
}

// One tensor's input and outputs must be disjoint (the kernels read x through the
// non-coherent path and write the outputs in the same pass).  Checked per tensor;
// overlaps between different tensors of a call are the caller's to avoid.
qf_status check_disjoint(const qf_tensor& t, int i, qf_format f, bool use_y, bool use_scales) {
    const int64_t n = t.rows * t.cols;
    const bool q4 = f == QF_Q4K || f == QF_Q4K_MSE;
    const int64_t nx = n * (t.x_type == QF_X_F32 ? 4 : 2);
    const int64_t ny = use_y ? n * 2 : 0;
    const int64_t nc = q4 ? n / 256 * 144 : n / 2;
    const int64_t ns = use_scales && !q4 ? n / block_of(f) : 0;
    const void* y = use_y ? t.y : nullptr;
    const void* sc = use_scales && !q4 ? t.scales : nullptr;
    if (overlap(t.x, nx, y, ny) || overlap(t.x, nx, t.codes, nc) || overlap(t.x, nx, sc, ns) ||
        overlap(y, ny, t.codes, nc) || overlap(y, ny, sc, ns) || overlap(t.codes, nc, sc, ns))
        return fail(QF_ERR_INVALID_ARG, "tensor %d: x, y, codes and scales must not overlap", i);
    return QF_OK;
}
bool known_format(qf_format f) {
    return f == QF_NVFP4 || f == QF_MXFP4 || f == QF_Q4K || f == QF_Q4K_MSE;
}

// Launch shape of one kernel: SM count, resident CTAs per SM, CTA size, waves.
struct Launch { int sms; int per_sm; int threads; int waves; };
// The SM count and occupancy of a (kernel, CTA size, device) are queried once per
// host thread and kept: the queries cost microseconds of host time per call.
struct ShapeEntry { const void* kernel; int threads; int dev; int sms; int per_sm; };

template <typename K>
qf_status launch_shape(K kernel, int threads, int waves, Launch* L) {
    thread_local std::vector<ShapeEntry> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    const void* key = reinterpret_cast<const void*>(kernel);
    L->threads = threads;
    L->waves = waves;
    for (const ShapeEntry& c : cache) {
        if (c.kernel == key && c.threads == threads && c.dev == dev) {
            L->sms = c.sms;
            L->per_sm = c.per_sm;
            return QF_OK;
        }
    }
    e = cudaDeviceGetAttribute(&L->sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&L->per_sm, kernel, threads, 0);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (L->per_sm < 1) L->per_sm = 1;
    cache.push_back({key, threads, dev, L->sms, L->per_sm});
    return QF_OK;
}

// Grid: one warp per unit, capped at `waves` CTAs per resident slot (1 = persistent).
int grid_for(const Launch& L, int64_t units) {
    const int64_t warps_per_cta = L.threads / 32;
    int64_t want = (units + warps_per_cta - 1) / warps_per_cta;
    int64_t cap = int64_t(L.sms) * L.per_sm * L.waves;
    return (int)std::max<int64_t>(1, std::min<int64_t>(std::min<int64_t>(want, cap), INT32_MAX));
}

template <int MAXT>
void fill_table(Table<MAXT>& P, const std::vector<DevTensor>& v, size_t begin, size_t count,
                int64_t unit_elems) {
    memset(&P, 0, sizeof P);
    int64_t u = 0;
    for (size_t i = 0; i < count; ++i) {
        DevTensor d = v[begin + i];
        d.unit_begin = u;
        u += (d.numel + unit_elems - 1) / unit_elems;
        d.unit_end = u;
        P.t[i] = d;
    }
    P.total_units = u;
    P.n = (int)count;
}

// Launch as a programmatic dependent of the previous kernel in the stream: this grid
// may start once every CTA of that one has run griddepcontrol.launch_dependents, and
// waits for its results with griddepcontrol.wait.
template <typename K, typename T>
cudaError_t launch_dependent(K kernel, unsigned grid, int threads, const T& P, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, P);
}

// Launch `kernel<MAXT>` over v in chunks of at most kLargeT tensors (as programmatic
// dependents of the previous kernel when `dependent`).
template <typename KS, typename KL>
qf_status launch_chunks(KS small_kernel, KL large_kernel, int threads, int waves,
                        const std::vector<DevTensor>& v, int64_t unit_elems, const float* amax,
                        float* scale_out, float* tracked, int n_groups, cudaStream_t s,
                        bool dependent = false, bool reverse = false) {
    Launch Ls, Ll;
    qf_status st = launch_shape(small_kernel, threads, waves, &Ls);
    if (st != QF_OK) return st;
    st = launch_shape(large_kernel, threads, waves, &Ll);
    if (st != QF_OK) return st;
    if (v.empty() && scale_out) {
        // nothing to quantize, but the per-group tensor scales are still reported
        Table<kSmallT> P;
        memset(&P, 0, sizeof P);
        P.group_amax = amax;
        P.group_scale_out = scale_out;
        P.n_groups = n_groups;
        small_kernel<<<1, threads, 0, s>>>(P);
    }
    for (size_t b = 0; b < v.size(); b += kLargeT) {
        const size_t cnt = std::min<size_t>(kLargeT, v.size() - b);
        float* so = b == 0 ? scale_out : nullptr;
        if (cnt <= (size_t)kSmallT) {
            Table<kSmallT> P;
            fill_table(P, v, b, cnt, unit_elems);
            P.group_amax = amax; P.group_scale_out = so; P.tracked = tracked; P.n_groups = n_groups;
            P.reverse = reverse;
            if (dependent) {
                cudaError_t e = launch_dependent(small_kernel, grid_for(Ls, P.total_units), threads, P, s);
                if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx");
            } else {
                small_kernel<<<grid_for(Ls, P.total_units), threads, 0, s>>>(P);
            }
        } else {
            Table<kLargeT> Q;              // ~27 KB kernel parameter
            fill_table(Q, v, b, cnt, unit_elems);
            Q.group_amax = amax; Q.group_scale_out = so; Q.tracked = tracked; Q.n_groups = n_groups;
            Q.reverse = reverse;
            if (dependent) {
                cudaError_t e = launch_dependent(large_kernel, grid_for(Ll, Q.total_units), threads, Q, s);
                if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx");
            } else {
                large_kernel<<<grid_for(Ll, Q.total_units), threads, 0, s>>>(Q);
            }
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return QF_OK;
}

// Validate one tensor; `need_cols_multiple` is 0 for qf_amax_tied.
qf_status check_tensor(const qf_tensor& t, int i, int need_cols_multiple, int n_groups,
                       bool check_group) {
    if (t.rows < 0 || t.cols < 0) return fail(QF_ERR_SHAPE, "tensor %d: negative size", i);
    if (t.cols > 0 && t.rows > INT64_MAX / 4 / t.cols)
        return fail(QF_ERR_SHAPE, "tensor %d: rows*cols overflows", i);
    if (need_cols_multiple && t.cols % need_cols_multiple != 0)
        return fail(QF_ERR_SHAPE, "tensor %d: cols=%lld is not a multiple of %d", i,
                    (long long)t.cols, need_cols_multiple);
    if (t.x_type != QF_X_BF16 && t.x_type != QF_X_F32)
        return fail(QF_ERR_UNSUPPORTED, "tensor %d: unknown x_type %d", i, (int)t.x_type);
    const int64_t numel = t.rows * t.cols;
    if (numel > 0 && t.x == nullptr) return fail(QF_ERR_INVALID_ARG, "tensor %d: x is NULL", i);
    if (!aligned16(t.x)) return fail(QF_ERR_ALIGN, "tensor %d: x not 16-byte aligned", i);
    if (check_group && (t.group < 0 || t.group >= n_groups))
        return fail(QF_ERR_INVALID_ARG, "tensor %d: group %d outside [0, %d)", i, t.group, n_groups);
    return QF_OK;
}

// The kernels of each format with their launch shapes (XT: input element type).
// FP32 input holds twice the bytes per element in registers: half the sub-tiles per unit
template <typename XT>
constexpr int nvb_u() { return sizeof(XT) == 2 ? QF_NVB_U : (QF_NVB_U + 1) / 2; }
template <typename XT, int MAXT>
constexpr auto nv_block_kernel() {
    return qf::k_nv<XT, nvb_u<XT>(), MAXT, QF_NVB_THREADS, QF_NVB_PREFETCH>;
}
template <typename XT, int MAXT, int MODE>
constexpr auto mx_kernel() {
    return qf::k_fp4<false, XT, kFp4U, MAXT, MODE, QF_MX_THREADS, QF_MX_PREFETCH>;
}
template <typename XT, bool MSE = false>
constexpr int q4k_threads() {
    return sizeof(XT) == 2 ? (MSE ? QF_Q4K_MSE_THREADS : QF_Q4K_THREADS) : QF_Q4K_F32_THREADS;
}
template <typename XT, int MAXT, int MODE, bool MSE>
constexpr auto q4k_kernel() {
    return qf::k_q4k<XT, MAXT, MODE, q4k_threads<XT, MSE>(), MSE>;
}

template <typename XT>
qf_status launch_format_t(qf_format f, int mode, const std::vector<DevTensor>& v,
                          const float* am, float* so, int ng, cudaStream_t s) {
    if (f == QF_NVFP4) {
        // the fused pass usually follows the tie-group amax pass over the same tensors:
        // from the last unit down, its first reads are still in L2
        if (mode == 0)
            return launch_chunks(nv_block_kernel<XT, kSmallT>(), nv_block_kernel<XT, kLargeT>(),
                                 QF_NVB_THREADS, QF_NVB_WAVES, v, 512 * nvb_u<XT>(), am, so, nullptr,
                                 ng, s, false, QF_NV_REVERSE);
        return launch_chunks(qf::k_nv_ste<XT, nvb_u<XT>(), kSmallT, QF_NVB_THREADS>,
                             qf::k_nv_ste<XT, nvb_u<XT>(), kLargeT, QF_NVB_THREADS>,
                             QF_NVB_THREADS, QF_NVB_WAVES, v, 512 * nvb_u<XT>(), am, nullptr,
                             nullptr, ng, s);
    }
    if (f == QF_MXFP4) {
        if (mode == 0)
            return launch_chunks(mx_kernel<XT, kSmallT, 0>(), mx_kernel<XT, kLargeT, 0>(), QF_MX_THREADS,
                                 QF_MX_WAVES, v, 256 * kFp4U, nullptr, nullptr, nullptr, 0, s);
        return launch_chunks(mx_kernel<XT, kSmallT, 1>(), mx_kernel<XT, kLargeT, 1>(), QF_MX_THREADS,
                             QF_MX_WAVES, v, 256 * kFp4U, nullptr, nullptr, nullptr, 0, s);
    }
    if (f == QF_Q4K_MSE) {
        if (mode == 0)
            return launch_chunks(q4k_kernel<XT, kSmallT, 0, true>(),
                                 q4k_kernel<XT, kLargeT, 0, true>(), q4k_threads<XT, true>(),
                                 QF_Q4K_WAVES, v, 1024, nullptr, nullptr, nullptr, 0, s);
        return launch_chunks(q4k_kernel<XT, kSmallT, 1, true>(), q4k_kernel<XT, kLargeT, 1, true>(),
                             q4k_threads<XT, true>(), QF_Q4K_WAVES, v, 1024, nullptr, nullptr,
                             nullptr, 0, s);
    }
    if (mode == 0)
        return launch_chunks(q4k_kernel<XT, kSmallT, 0, false>(),
                             q4k_kernel<XT, kLargeT, 0, false>(), q4k_threads<XT>(), QF_Q4K_WAVES, v,
                             1024, nullptr, nullptr, nullptr, 0, s);
    return launch_chunks(q4k_kernel<XT, kSmallT, 1, false>(), q4k_kernel<XT, kLargeT, 1, false>(),
                         q4k_threads<XT>(), QF_Q4K_WAVES, v, 1024, nullptr, nullptr, nullptr, 0, s);
}

qf_status launch_format(qf_format f, int mode, int x_type, const std::vector<DevTensor>& v,
                        const float* am, float* so, int ng, cudaStream_t s) {
    if (x_type == QF_X_F32) return launch_format_t<float>(f, mode, v, am, so, ng, s);
    return launch_format_t<uint16_t>(f, mode, v, am, so, ng, s);
}

qf_status fakequant_impl(qf_format f, const qf_tensor* t, int n, const float* d_group_amax,
                         int n_groups, float* d_group_scale_out, void* stream, bool pack_only) {
    g_err[0] = 0;
    if (!known_format(f)) return fail(QF_ERR_UNSUPPORTED, "unknown format %d", (int)f);
    if (n < 0) return fail(QF_ERR_INVALID_ARG, "n = %d < 0", n);
    if (n > 0 && t == nullptr) return fail(QF_ERR_INVALID_ARG, "tensor array is NULL");
    const bool nv = f == QF_NVFP4;
    if (nv) {
        if (n_groups <= 0) return fail(QF_ERR_INVALID_ARG, "NVFP4 needs n_groups > 0");
        if (d_group_amax == nullptr) return fail(QF_ERR_INVALID_ARG, "NVFP4 needs d_group_amax");
    }
    std::vector<DevTensor> v;
    v.reserve(n);
    for (int i = 0; i < n; ++i) {
        qf_status st = check_tensor(t[i], i, block_of(f), n_groups, nv);
        if (st != QF_OK) return st;
        const int64_t numel = t[i].rows * t[i].cols;
        if (numel == 0) continue;
        void* y = pack_only ? nullptr : t[i].y;
        void* scales = (f == QF_Q4K || f == QF_Q4K_MSE) ? nullptr : t[i].scales;
        if (!y && !t[i].codes && !scales)
            return fail(QF_ERR_INVALID_ARG, "tensor %d: no output (y, codes, scales all NULL)", i);
        if (!aligned16(y) || !aligned16(t[i].codes))
            return fail(QF_ERR_ALIGN, "tensor %d: y / codes not 16-byte aligned", i);
        st = check_disjoint(t[i], i, f, !pack_only, true);
        if (st != QF_OK) return st;
        DevTensor d{};
        if (t[i].x_type != t[0].x_type)
            return fail(QF_ERR_INVALID_ARG, "tensor %d: x_type differs from tensor 0's", i);
        d.x = t[i].x;
        d.y = static_cast<uint16_t*>(y);
        d.codes = static_cast<uint8_t*>(t[i].codes);
        d.scales = static_cast<uint8_t*>(scales);
        d.numel = numel;
        d.group = nv ? t[i].group : 0;
        v.push_back(d);
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* so = nv ? d_group_scale_out : nullptr;
    const float* am = nv ? d_group_amax : nullptr;
    const int ng = nv ? n_groups : 0;
    if (v.empty() && !so) return QF_OK;
    return launch_format(f, 0, n > 0 ? t[0].x_type : QF_X_BF16, v, am, so, ng, s);
}

// ------------------------------------------------------------------ LoRA
constexpr int kLoraSmallT = 8;
constexpr int kLoraLargeT = 256;

template <int MODE, int R>
qf_status lora_launch_r(const std::vector<qf::LoraTensor>& v, const float* am, float* so, int ng,
                        cudaStream_t s) {
    // merge modes and NVFP4 up to rank 16: 8 columns per lane (k_lora8), kLora8Rows-row units
    constexpr bool k8 = QF_LORA8 && R <= 16 &&
                        (MODE == qf::kLoraMerge || MODE == qf::kLoraMergeAmax ||
                         (QF_LORA8_NV && MODE == qf::kLoraNV));
    constexpr int64_t kRowsPerUnit = k8 ? qf::kLora8Rows : qf::kLoraRows;
    for (size_t b = 0; b < v.size(); b += kLoraLargeT) {
        const size_t cnt = std::min<size_t>(kLoraLargeT, v.size() - b);
        float* sout = b == 0 ? so : nullptr;
        auto fill = [&](auto& P) {
            memset(&P, 0, sizeof P);
            int64_t u = 0;
            for (size_t i = 0; i < cnt; ++i) {
                qf::LoraTensor d = v[b + i];
                d.unit_begin = u;
                u += ((d.rows + kRowsPerUnit - 1) / kRowsPerUnit) * d.col_groups;
                P.t[i] = d;
            }
            P.total_units = u;
            P.n = (int)cnt;
            P.group_amax = am;
            P.group_scale_out = sout;
            P.n_groups = ng;
        };
        if (cnt <= (size_t)kLoraSmallT) {
            qf::LoraTable<kLoraSmallT> P;
            fill(P);
            const unsigned grid = (unsigned)std::max<int64_t>(1, P.total_units);
            if constexpr (k8) qf::k_lora8<MODE, R, kLoraSmallT><<<grid, qf::kLora8Threads, 0, s>>>(P);
            else qf::k_lora<MODE, R, kLoraSmallT><<<grid, qf::kLoraThreads, 0, s>>>(P);
        } else {
            qf::LoraTable<kLoraLargeT> P;
            fill(P);
            const unsigned grid = (unsigned)std::max<int64_t>(1, P.total_units);
            if constexpr (k8) qf::k_lora8<MODE, R, kLoraLargeT><<<grid, qf::kLora8Threads, 0, s>>>(P);
            else qf::k_lora<MODE, R, kLoraLargeT><<<grid, qf::kLoraThreads, 0, s>>>(P);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    }
    return QF_OK;
}

// k_lora_amax over the tensors of a call (units of kLoraAmaxRows rows x kLoraCols
// columns); folds each tie group's exact max |M| into d_group_amax, which must hold
// exact values only (zeros, or an earlier fold of the same group).
qf_status lora_amax_launch(const std::vector<qf::LoraTensor>& v, float* am, cudaStream_t s) {
    for (size_t b = 0; b < v.size(); b += kLoraLargeT) {
        const size_t cnt = std::min<size_t>(kLoraLargeT, v.size() - b);
        auto fill = [&](auto& P) {
            memset(&P, 0, sizeof P);
            int64_t u = 0;
            for (size_t i = 0; i < cnt; ++i) {
                qf::LoraTensor d = v[b + i];
                d.unit_begin = u;
                u += ((d.rows + qf::kLoraAmaxRows - 1) / qf::kLoraAmaxRows) * d.col_groups;
                P.t[i] = d;
            }
            P.total_units = u;
            P.n = (int)cnt;
            P.group_amax = am;
        };
        if (cnt <= (size_t)kLoraSmallT) {
            qf::LoraTable<kLoraSmallT> P;
            fill(P);
            qf::k_lora_amax<kLoraSmallT>
                <<<(unsigned)std::max<int64_t>(1, P.total_units), qf::kLoraThreads, 0, s>>>(P);
        } else {
            qf::LoraTable<kLoraLargeT> P;
            fill(P);
            qf::k_lora_amax<kLoraLargeT>
                <<<(unsigned)std::max<int64_t>(1, P.total_units), qf::kLoraThreads, 0, s>>>(P);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    }
    return QF_OK;
}

template <int MODE>
qf_status lora_launch(const std::vector<qf::LoraTensor>& v, int max_rank, const float* am,
                      float* so, int ng, cudaStream_t s) {
    if (max_rank <= 8) return lora_launch_r<MODE, 8>(v, am, so, ng, s);
    if (max_rank <= 16) return lora_launch_r<MODE, 16>(v, am, so, ng, s);
    return lora_launch_r<MODE, 32>(v, am, so, ng, s);
}

// Validate and describe the (tensor, adapter) pairs of a LoRA call.
qf_status lora_tensors(const qf_tensor* t, const qf_lora* l, int n, int cols_multiple,
                       int n_groups, bool check_group, bool need_output,
                       std::vector<qf::LoraTensor>* out, int* max_rank) {
    if (n < 0) return fail(QF_ERR_INVALID_ARG, "n = %d < 0", n);
    if (n > 0 && (t == nullptr || l == nullptr))
        return fail(QF_ERR_INVALID_ARG, "tensor or adapter array is NULL");
    *max_rank = 1;
    for (int i = 0; i < n; ++i) {
        qf_status st = check_tensor(t[i], i, cols_multiple, n_groups, check_group);
        if (st != QF_OK) return st;
        if (t[i].x_type != QF_X_BF16)
            return fail(QF_ERR_UNSUPPORTED, "tensor %d: LoRA bases are BF16", i);
        if (l[i].rank < 1 || l[i].rank > QF_LORA_MAX_RANK)
            return fail(QF_ERR_INVALID_ARG, "tensor %d: rank %d outside [1, %d]", i, l[i].rank,
                        QF_LORA_MAX_RANK);
        const int64_t numel = t[i].rows * t[i].cols;
        if (numel == 0) continue;
        if (l[i].a == nullptr || l[i].b == nullptr)
            return fail(QF_ERR_INVALID_ARG, "tensor %d: adapter a / b is NULL", i);
        if (!aligned16(l[i].a)) return fail(QF_ERR_ALIGN, "tensor %d: adapter a not 16-byte aligned", i);
        if ((reinterpret_cast<uintptr_t>(l[i].b) & 1u) != 0)
            return fail(QF_ERR_ALIGN, "tensor %d: adapter b not 2-byte aligned", i);
        if (need_output && !t[i].y && !t[i].codes && !t[i].scales)
            return fail(QF_ERR_INVALID_ARG, "tensor %d: no output", i);
        if (!aligned16(t[i].y) || !aligned16(t[i].codes))
            return fail(QF_ERR_ALIGN, "tensor %d: y / codes not 16-byte aligned", i);
        st = check_disjoint(t[i], i, cols_multiple == 32 ? QF_MXFP4 : QF_NVFP4, true, true);
        if (st != QF_OK) return st;
        qf::LoraTensor d{};
        d.w = static_cast<const uint16_t*>(t[i].x);
        d.b = static_cast<const uint16_t*>(l[i].b);
        d.a = static_cast<const uint16_t*>(l[i].a);
        d.y = static_cast<uint16_t*>(t[i].y);
        d.codes = static_cast<uint8_t*>(t[i].codes);
        d.scales = static_cast<uint8_t*>(t[i].scales);
        d.rows = t[i].rows;
        d.cols = t[i].cols;
        d.col_groups = (t[i].cols + qf::kLoraCols - 1) / qf::kLoraCols;
        d.rank = l[i].rank;
        d.scale = l[i].scale;
        d.group = check_group ? t[i].group : 0;
        *max_rank = std::max(*max_rank, (int)l[i].rank);
        out->push_back(d);
    }
    return QF_OK;
}

// Zero the group amax, then fold max |x| of every tensor into its group (and into
// the running amax when d_tracked is given).
qf_status amax_launch(const std::vector<DevTensor>& v, int x_type, float* d_group_amax,
                      int n_groups, float* d_tracked, cudaStream_t s) {
    bool ragged = false;
    for (const DevTensor& d : v) ragged |= (d.numel & 7) != 0;
    cudaError_t e = cudaMemsetAsync(d_group_amax, 0, sizeof(float) * (size_t)n_groups, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    if (v.empty()) return QF_OK;
    const bool f32 = x_type == QF_X_F32;
    // the same bytes in flight per lane: 8 vectors of BF16, or 4 sub-tiles of FP32 (8 vectors)
    qf_status st = f32
        ? launch_chunks(qf::k_amax<float, kAmaxU / 2, kSmallT, QF_AMAX_THREADS>,
                        qf::k_amax<float, kAmaxU / 2, kLargeT, QF_AMAX_THREADS>, QF_AMAX_THREADS,
                        QF_AMAX_WAVES, v, 256 * (kAmaxU / 2), d_group_amax, nullptr, d_tracked,
                        n_groups, s)
        : launch_chunks(qf::k_amax<uint16_t, kAmaxU, kSmallT, QF_AMAX_THREADS>,
                        qf::k_amax<uint16_t, kAmaxU, kLargeT, QF_AMAX_THREADS>, QF_AMAX_THREADS,
                        QF_AMAX_WAVES, v, 256 * kAmaxU, d_group_amax, nullptr, d_tracked,
                        n_groups, s);
    if (st != QF_OK || !ragged) return st;
    // scalar tails of tensors whose size is not a multiple of 8 elements
    for (size_t b = 0; b < v.size(); b += kSmallT) {
        const size_t cnt = std::min<size_t>(kSmallT, v.size() - b);
        Table<kSmallT> P;
        fill_table(P, v, b, cnt, 256 * kAmaxU);
        P.group_amax = d_group_amax;
        P.tracked = d_tracked;
        P.n_groups = n_groups;
        if (f32) qf::k_amax_tail<float, kSmallT><<<(unsigned)cnt, 32, 0, s>>>(P);
        else qf::k_amax_tail<uint16_t, kSmallT><<<(unsigned)cnt, 32, 0, s>>>(P);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return QF_OK;
}

// ------------------------------------------------------------------ one-shot NVFP4
constexpr size_t oneshot_ws_bytes(int n_groups) {
    return (sizeof(uint32_t) * ((size_t)qf::kOneshotHeaderWords + (size_t)n_groups) + 255) / 256 *
           256;
}

// Polls of the forced barrier timeout (qf_test_barrier_timeout); 0 = normal operation.
std::atomic<uint32_t> g_test_polls{0};

// L2 size and cooperative-launch support of the current device, queried once per
// host thread and device.
struct DevProps { int dev; int l2; int coop; };
qf_status dev_props(DevProps* D) {
    thread_local std::vector<DevProps> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    for (const DevProps& c : cache) {
        if (c.dev == dev) {
            *D = c;
            return QF_OK;
        }
    }
    DevProps d{dev, 0, 0};
    e = cudaDeviceGetAttribute(&d.l2, cudaDevAttrL2CacheSize, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    e = cudaDeviceGetAttribute(&d.coop, cudaDevAttrCooperativeLaunch, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    cache.push_back(d);
    *D = d;
    return QF_OK;
}

template <typename XT, int MAXT>
qf_status oneshot_launch(const std::vector<DevTensor>& v, float* am, float* tracked, float* so,
                         int ng, uint32_t* ws, cudaStream_t s) {
    constexpr int U = nvb_u<XT>();
    auto kernel = qf::k_nv_oneshot<XT, U, MAXT, QF_ONESHOT_THREADS>;
    Launch L;
    qf_status st = launch_shape(kernel, QF_ONESHOT_THREADS, 1, &L);
    if (st != QF_OK) return st;
    Table<MAXT> P;
    fill_table(P, v, 0, v.size(), 512 * U);
    P.group_amax = am;
    P.tracked = tracked;
    P.group_scale_out = so;
    P.n_groups = ng;
    // at most one CTA per resident slot: every CTA must be resident for the barrier,
    // which the cooperative launch guarantees (or refuses to launch)
    const int grid = grid_for(L, P.total_units);
    uint32_t test_polls = g_test_polls.load(std::memory_order_relaxed);
    void* args[] = {&P, &ws, &test_polls};
    cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel), dim3(grid),
                                                dim3(QF_ONESHOT_THREADS), args, 0, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchCooperativeKernel");
    return QF_OK;
}

// ------------------------------------------------------------------ static scratch
// The workspace of qf_amax_fakequant_noalloc: module-level device memory, one copy per
// device, never allocated at run time.  Capacity: the workspace qf_amax_fakequant needs
// for QF_NOALLOC_MAX_GROUPS tie groups (header words plus one word per group, rounded
// up to 256 bytes), so every byte a call clears or uses lies inside the array.
constexpr size_t kNoallocBytes = oneshot_ws_bytes(QF_NOALLOC_MAX_GROUPS);
static_assert(kNoallocBytes % sizeof(uint32_t) == 0, "whole words");
__device__ __align__(256) uint32_t g_noalloc_ws[kNoallocBytes / sizeof(uint32_t)];

// Its address on the current device, looked up once per device (with that device
// current, as cudaGetSymbolAddress requires) and kept.
qf_status noalloc_ws(void** out) {
    static std::mutex mu;
    static std::vector<std::pair<int, void*>> addr;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lock(mu);
    for (const auto& a : addr) {
        if (a.first == dev) {
            *out = a.second;
            return QF_OK;
        }
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_ws);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
    addr.emplace_back(dev, p);
    *out = p;
    return QF_OK;
}

}  // namespace

extern "C" {

qf_status qf_lora_merge(const qf_tensor* t, const qf_lora* l, int n, void* stream) {
    g_err[0] = 0;
    std::vector<qf::LoraTensor> v;
    int max_rank;
    qf_status st = lora_tensors(t, l, n, 16, 0, false, false, &v, &max_rank);
    if (st != QF_OK) return st;
    for (int i = 0; i < n; ++i)
        if (t[i].rows * t[i].cols > 0 && t[i].y == nullptr)
            return fail(QF_ERR_INVALID_ARG, "tensor %d: y (the merged output) is NULL", i);
    if (v.empty()) return QF_OK;
    return lora_launch<qf::kLoraMerge>(v, max_rank, nullptr, nullptr, 0,
                                       static_cast<cudaStream_t>(stream));
}

qf_status qf_amax_tied_lora(const qf_tensor* t, const qf_lora* l, int n, float* d_group_amax,
                            int n_groups, void* stream) {
    g_err[0] = 0;
    if (n_groups <= 0) return fail(QF_ERR_INVALID_ARG, "n_groups = %d <= 0", n_groups);
    if (d_group_amax == nullptr) return fail(QF_ERR_INVALID_ARG, "d_group_amax is NULL");
    std::vector<qf::LoraTensor> v;
    int max_rank;
    qf_status st = lora_tensors(t, l, n, 16, n_groups, true, false, &v, &max_rank);
    if (st != QF_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(d_group_amax, 0, sizeof(float) * (size_t)n_groups, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    if (v.empty()) return QF_OK;
    return lora_amax_launch(v, d_group_amax, s);
}

qf_status qf_fakequant_lora(qf_format f, const qf_tensor* t, const qf_lora* l, int n,
                            const float* d_group_amax, int n_groups, float* d_group_scale_out,
                            void* stream) {
    g_err[0] = 0;
    if (f != QF_NVFP4 && f != QF_MXFP4)
        return fail(QF_ERR_UNSUPPORTED, "qf_fakequant_lora fuses NVFP4 and MXFP4 (got %d)", (int)f);
    const bool nv = f == QF_NVFP4;
    if (nv && (n_groups <= 0 || d_group_amax == nullptr))
        return fail(QF_ERR_INVALID_ARG, "NVFP4 needs d_group_amax and n_groups > 0");
    std::vector<qf::LoraTensor> v;
    int max_rank;
    qf_status st = lora_tensors(t, l, n, nv ? 16 : 32, n_groups, nv, true, &v, &max_rank);
    if (st != QF_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* so = nv ? d_group_scale_out : nullptr;
    if (v.empty() && !so) return QF_OK;
    if (v.empty()) {
        // nothing to quantize; still report the tensor scales
        qf::LoraTensor none{};
        none.rows = 0;
        none.cols = 16;
        none.col_groups = 1;
        none.rank = 1;
        v.push_back(none);
    }
    if (nv) return lora_launch<qf::kLoraNV>(v, max_rank, d_group_amax, so, n_groups, s);
    return lora_launch<qf::kLoraMX>(v, max_rank, nullptr, nullptr, 0, s);
}


qf_status qf_amax_fakequant_lora(const qf_tensor* t, const qf_lora* l, int n,
                                 float* d_group_amax, int n_groups, float* d_group_scale_out,
                                 void* stream) {
    g_err[0] = 0;
    if (n_groups <= 0) return fail(QF_ERR_INVALID_ARG, "n_groups = %d <= 0", n_groups);
    if (d_group_amax == nullptr) return fail(QF_ERR_INVALID_ARG, "d_group_amax is NULL");
    std::vector<qf::LoraTensor> v;
    int max_rank;
    qf_status st = lora_tensors(t, l, n, 16, n_groups, true, true, &v, &max_rank);
    if (st != QF_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(d_group_amax, 0, sizeof(float) * (size_t)n_groups, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    bool all_y = true;
    for (const qf::LoraTensor& d : v) all_y &= d.y != nullptr;
    // With room for it in y, the merged weight is written once with its amax and
    // quantized in place.  Otherwise (or with QF_LORA_STEP_TWO_PASS up to rank 16) the
    // step reads W twice: the pruned exact amax, then the merge-on-the-fly NVFP4 pass.
    const bool two_pass = v.empty() || !all_y || (QF_LORA_STEP_TWO_PASS && max_rank <= 16);
    if (two_pass) {
        if (!v.empty()) {
            st = lora_amax_launch(v, d_group_amax, s);
            if (st != QF_OK) return st;
        }
        if (v.empty() && !d_group_scale_out) return QF_OK;
        if (v.empty()) {
            qf::LoraTensor none{};
            none.rows = 0;
            none.cols = 16;
            none.col_groups = 1;
            none.rank = 1;
            v.push_back(none);
        }
        return lora_launch<qf::kLoraNV>(v, max_rank, d_group_amax, d_group_scale_out, n_groups, s);
    }
    // the merged weight is formed once, written into y with its group amax, and y is
    // then quantized in place by the plain NVFP4 pass (every lane reads its block
    // before it writes it, and blocks are disjoint)
    st = lora_launch<qf::kLoraMergeAmax>(v, max_rank, d_group_amax, nullptr, n_groups, s);
    if (st != QF_OK) return st;
    std::vector<DevTensor> w;
    w.reserve(v.size());
    for (const qf::LoraTensor& d : v) {
        DevTensor x{};
        x.x = d.y;
        x.y = d.y;
        x.codes = d.codes;
        x.scales = d.scales;
        x.numel = d.rows * d.cols;
        x.group = d.group;
        w.push_back(x);
    }
    // coherent loads: this pass writes the buffer it reads
    return launch_chunks(qf::k_nv<uint16_t, nvb_u<uint16_t>(), kSmallT, QF_NVB_THREADS,
                                  QF_NVB_PREFETCH, 3>,
                         qf::k_nv<uint16_t, nvb_u<uint16_t>(), kLargeT, QF_NVB_THREADS,
                                  QF_NVB_PREFETCH, 3>,
                         QF_NVB_THREADS, QF_NVB_WAVES, w, 512 * nvb_u<uint16_t>(), d_group_amax,
                         d_group_scale_out, nullptr, n_groups, s, false, QF_NV_REVERSE);
}

qf_status qf_amax_tied(const qf_tensor* t, int n, float* d_group_amax, int n_groups,
                       float* d_tracked, void* stream) {
    g_err[0] = 0;
    if (n < 0) return fail(QF_ERR_INVALID_ARG, "n = %d < 0", n);
    if (n > 0 && t == nullptr) return fail(QF_ERR_INVALID_ARG, "tensor array is NULL");
    if (n_groups <= 0) return fail(QF_ERR_INVALID_ARG, "n_groups = %d <= 0", n_groups);
    if (d_group_amax == nullptr) return fail(QF_ERR_INVALID_ARG, "d_group_amax is NULL");
    std::vector<DevTensor> v;
    for (int i = 0; i < n; ++i) {
        qf_status st = check_tensor(t[i], i, 0, n_groups, true);
        if (st != QF_OK) return st;
        if (t[i].x_type != t[0].x_type)
            return fail(QF_ERR_INVALID_ARG, "tensor %d: x_type differs from tensor 0's", i);
        const int64_t numel = t[i].rows * t[i].cols;
        if (numel == 0) continue;
        DevTensor d{};
        d.x = t[i].x;
        d.numel = numel;
        d.group = t[i].group;
        v.push_back(d);
    }
    return amax_launch(v, n > 0 ? t[0].x_type : QF_X_BF16, d_group_amax, n_groups, d_tracked,
                       static_cast<cudaStream_t>(stream));
}

size_t qf_amax_fakequant_workspace_bytes(int n_groups) {
    return n_groups > 0 ? oneshot_ws_bytes(n_groups) : 0;
}

qf_status qf_amax_fakequant(const qf_tensor* t, int n, float* d_group_amax, int n_groups,
                            float* d_tracked, float* d_group_scale_out, void* d_workspace,
                            size_t workspace_bytes, void* stream) {
    g_err[0] = 0;
    if (n < 0) return fail(QF_ERR_INVALID_ARG, "n = %d < 0", n);
    if (n > 0 && t == nullptr) return fail(QF_ERR_INVALID_ARG, "tensor array is NULL");
    if (n_groups <= 0) return fail(QF_ERR_INVALID_ARG, "n_groups = %d <= 0", n_groups);
    if (d_group_amax == nullptr) return fail(QF_ERR_INVALID_ARG, "d_group_amax is NULL");
    if (d_workspace != nullptr) {
        if (workspace_bytes < oneshot_ws_bytes(n_groups))
            return fail(QF_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed for %d groups",
                        workspace_bytes, oneshot_ws_bytes(n_groups), n_groups);
        if (!aligned16(d_workspace)) return fail(QF_ERR_ALIGN, "workspace not 16-byte aligned");
    }
    // every check of qf_amax_tied and of qf_fakequant(QF_NVFP4) before anything launches
    std::vector<DevTensor> v;
    v.reserve(n);
    int64_t in_bytes = 0;
    for (int i = 0; i < n; ++i) {
        qf_status st = check_tensor(t[i], i, 16, n_groups, true);
        if (st != QF_OK) return st;
        if (t[i].x_type != t[0].x_type)
            return fail(QF_ERR_INVALID_ARG, "tensor %d: x_type differs from tensor 0's", i);
        const int64_t numel = t[i].rows * t[i].cols;
        if (numel == 0) continue;
        if (!t[i].y && !t[i].codes && !t[i].scales)
            return fail(QF_ERR_INVALID_ARG, "tensor %d: no output (y, codes, scales all NULL)", i);
        if (!aligned16(t[i].y) || !aligned16(t[i].codes))
            return fail(QF_ERR_ALIGN, "tensor %d: y / codes not 16-byte aligned", i);
        st = check_disjoint(t[i], i, QF_NVFP4, true, true);
        if (st != QF_OK) return st;
        DevTensor d{};
        d.x = t[i].x;
        d.y = static_cast<uint16_t*>(t[i].y);
        d.codes = static_cast<uint8_t*>(t[i].codes);
        d.scales = static_cast<uint8_t*>(t[i].scales);
        d.numel = numel;
        d.group = t[i].group;
        v.push_back(d);
        in_bytes += numel * (t[i].x_type == QF_X_F32 ? 4 : 2);
    }
    const int x_type = n > 0 ? t[0].x_type : QF_X_BF16;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DevProps D;
    qf_status st = dev_props(&D);
    if (st != QF_OK) return st;
    const bool one = d_workspace != nullptr && !v.empty() && v.size() <= (size_t)kLargeT &&
                     D.coop && in_bytes * QF_ONESHOT_L2_DIV <= (int64_t)D.l2;
    if (one) {
        uint32_t* ws = static_cast<uint32_t*>(d_workspace);
        if (v.size() <= (size_t)kSmallT)
            return x_type == QF_X_F32
                ? oneshot_launch<float, kSmallT>(v, d_group_amax, d_tracked, d_group_scale_out,
                                                 n_groups, ws, s)
                : oneshot_launch<uint16_t, kSmallT>(v, d_group_amax, d_tracked, d_group_scale_out,
                                                    n_groups, ws, s);
        return x_type == QF_X_F32
            ? oneshot_launch<float, kLargeT>(v, d_group_amax, d_tracked, d_group_scale_out, n_groups,
                                             ws, s)
            : oneshot_launch<uint16_t, kLargeT>(v, d_group_amax, d_tracked, d_group_scale_out,
                                                n_groups, ws, s);
    }
    // two launches: the tie-group amax, then the fused pass on the scale it gives, as a
    // programmatic dependent of the amax grid (its first loads overlap that grid's end)
    st = amax_launch(v, x_type, d_group_amax, n_groups, d_tracked, s);
    if (st != QF_OK) return st;
    if (v.empty() && !d_group_scale_out) return QF_OK;
    const float* am = d_tracked ? d_tracked : d_group_amax;
    // grouped launches over many tensors measured slower as dependents (their early
    // loads compete with the amax grid's long tail): plain stream order for those
    if (v.empty() || v.size() > (size_t)kSmallT)
        return launch_format(QF_NVFP4, 0, x_type, v, am, d_group_scale_out, n_groups, s);
    if (x_type == QF_X_F32)
        return launch_chunks(qf::k_nv<float, nvb_u<float>(), kSmallT, QF_NVB_THREADS,
                                      QF_NVB_PREFETCH, QF_FP4_LD, true>,
                             qf::k_nv<float, nvb_u<float>(), kLargeT, QF_NVB_THREADS,
                                      QF_NVB_PREFETCH, QF_FP4_LD, true>,
                             QF_NVB_THREADS, QF_NVB_WAVES, v, 512 * nvb_u<float>(), am,
                             d_group_scale_out, nullptr, n_groups, s, true, QF_NV_REVERSE);
    return launch_chunks(qf::k_nv<uint16_t, nvb_u<uint16_t>(), kSmallT, QF_NVB_THREADS,
                                  QF_NVB_PREFETCH, QF_FP4_LD, true>,
                         qf::k_nv<uint16_t, nvb_u<uint16_t>(), kLargeT, QF_NVB_THREADS,
                                  QF_NVB_PREFETCH, QF_FP4_LD, true>,
                         QF_NVB_THREADS, QF_NVB_WAVES, v, 512 * nvb_u<uint16_t>(), am,
                         d_group_scale_out, nullptr, n_groups, s, true, QF_NV_REVERSE);
}

qf_status qf_amax_fakequant_noalloc(const qf_tensor* t, int n, float* d_group_amax,
                                    int n_groups, float* d_tracked, float* d_group_scale_out,
                                    void* stream) {
    g_err[0] = 0;
    if (n_groups > QF_NOALLOC_MAX_GROUPS)
        return fail(QF_ERR_INVALID_ARG, "n_groups = %d exceeds the static workspace (%d groups)",
                    n_groups, QF_NOALLOC_MAX_GROUPS);
    if (n_groups <= 0) return fail(QF_ERR_INVALID_ARG, "n_groups = %d <= 0", n_groups);
    // the argument checks of qf_amax_fakequant, made here too so that an invalid call
    // enqueues nothing (not even the clearing of the workspace)
    if (n < 0) return fail(QF_ERR_INVALID_ARG, "n = %d < 0", n);
    if (n > 0 && t == nullptr) return fail(QF_ERR_INVALID_ARG, "tensor array is NULL");
    if (d_group_amax == nullptr) return fail(QF_ERR_INVALID_ARG, "d_group_amax is NULL");
    for (int i = 0; i < n; ++i) {
        qf_status st = check_tensor(t[i], i, 16, n_groups, true);
        if (st != QF_OK) return st;
        if (t[i].x_type != t[0].x_type)
            return fail(QF_ERR_INVALID_ARG, "tensor %d: x_type differs from tensor 0's", i);
        if (t[i].rows * t[i].cols == 0) continue;
        if (!t[i].y && !t[i].codes && !t[i].scales)
            return fail(QF_ERR_INVALID_ARG, "tensor %d: no output (y, codes, scales all NULL)", i);
        if (!aligned16(t[i].y) || !aligned16(t[i].codes))
            return fail(QF_ERR_ALIGN, "tensor %d: y / codes not 16-byte aligned", i);
        st = check_disjoint(t[i], i, QF_NVFP4, true, true);
        if (st != QF_OK) return st;
    }
    void* ws = nullptr;
    qf_status st = noalloc_ws(&ws);
    if (st != QF_OK) return st;
    // the counters and slots this call uses must start at zero: clear them on the call's
    // stream, whatever an earlier call left there.  The error word (word 0) is kept: a
    // timeout stays visible to qf_noalloc_check until that call clears it.
    const size_t bytes = oneshot_ws_bytes(n_groups);
    constexpr size_t kKeep = sizeof(uint32_t);              // the error word
    cudaError_t e = cudaMemsetAsync(static_cast<char*>(ws) + kKeep, 0, bytes - kKeep,
                                    static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    return qf_amax_fakequant(t, n, d_group_amax, n_groups, d_tracked, d_group_scale_out, ws, bytes,
                             stream);
}

// Synchronizes `stream`, then reads the error word of a one-shot workspace and clears it.
static qf_status check_and_clear(const void* d_workspace, void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    uint32_t* word = static_cast<uint32_t*>(const_cast<void*>(d_workspace)) + qf::kOneshotErrWord;
    uint32_t err = 0;
    e = cudaMemcpy(&err, word, sizeof err, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
    if (err == 0) return QF_OK;
    const uint32_t zero = 0;
    e = cudaMemcpy(word, &zero, sizeof zero, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
    if (err & qf::kOneshotErrTimeout)
        return fail(QF_ERR_TIMEOUT, "a grid barrier gave up waiting; that call (and any later "
                                    "call on this workspace before this check) wrote no outputs");
    return fail(QF_ERR_CUDA, "unknown workspace error flags %#x", err);
}

qf_status qf_workspace_check(const void* d_workspace, void* stream) {
    g_err[0] = 0;
    if (d_workspace == nullptr) return fail(QF_ERR_INVALID_ARG, "workspace is NULL");
    return check_and_clear(d_workspace, stream);
}

qf_status qf_noalloc_check(void* stream) {
    g_err[0] = 0;
    void* ws = nullptr;
    qf_status st = noalloc_ws(&ws);
    if (st != QF_OK) return st;
    return check_and_clear(ws, stream);
}

void qf_test_barrier_timeout(unsigned int polls) {
    g_test_polls.store(polls, std::memory_order_relaxed);
}

qf_status qf_fakequant(qf_format f, const qf_tensor* t, int n, const float* d_group_amax,
                       int n_groups, float* d_group_scale_out, void* stream) {
    return fakequant_impl(f, t, n, d_group_amax, n_groups, d_group_scale_out, stream, false);
}

qf_status qf_pack(qf_format f, const qf_tensor* t, int n, const float* d_group_amax,
                  int n_groups, float* d_group_scale_out, void* stream) {
    return fakequant_impl(f, t, n, d_group_amax, n_groups, d_group_scale_out, stream, true);
}

qf_status qf_ste_backward(qf_format f, const void* grad_y, void* grad_x, int64_t numel, int mode,
                          const qf_tensor* fwd, const float* d_group_amax, int n_groups,
                          void* stream) {
    g_err[0] = 0;
    if (mode != 0 && mode != 1) return fail(QF_ERR_UNSUPPORTED, "unknown STE mode %d", mode);
    if (numel < 0) return fail(QF_ERR_SHAPE, "numel = %lld < 0", (long long)numel);
    if (numel > 0 && (grad_y == nullptr || grad_x == nullptr))
        return fail(QF_ERR_INVALID_ARG, "grad_y / grad_x is NULL");
    if (!aligned16(grad_y) || !aligned16(grad_x))
        return fail(QF_ERR_ALIGN, "grad_y / grad_x not 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (mode == 0) {
        if (numel == 0 || grad_x == grad_y) return QF_OK;
        if (overlap(grad_y, numel * 2, grad_x, numel * 2))
            return fail(QF_ERR_INVALID_ARG, "grad_x overlaps grad_y without being equal to it");
        const int64_t vec = numel / 8;
        const int grid = (int)std::max<int64_t>(1, (vec + 4 * kThreads - 1) / (4 * kThreads));
        qf::k_copy<<<grid, kThreads, 0, s>>>(static_cast<const uint16_t*>(grad_y),
                                             static_cast<uint16_t*>(grad_x), numel);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
        return QF_OK;
    }
    if (!known_format(f)) return fail(QF_ERR_UNSUPPORTED, "unknown format %d", (int)f);
    if (fwd == nullptr) return fail(QF_ERR_INVALID_ARG, "clipped STE needs the forward tensor");
    const bool nv = f == QF_NVFP4;
    if (nv && (n_groups <= 0 || d_group_amax == nullptr))
        return fail(QF_ERR_INVALID_ARG, "NVFP4 clipped STE needs d_group_amax and n_groups > 0");
    qf_status st = check_tensor(*fwd, 0, block_of(f), n_groups, nv);
    if (st != QF_OK) return st;
    if (fwd->rows * fwd->cols != numel)
        return fail(QF_ERR_SHAPE, "numel %lld != rows*cols of the forward tensor",
                    (long long)numel);
    // grad_x == grad_y is allowed: each element is read before the same thread writes it
    if (numel == 0) return QF_OK;
    std::vector<DevTensor> v(1);
    v[0] = DevTensor{};
    v[0].x = fwd->x;
    v[0].g = static_cast<const uint16_t*>(grad_y);
    v[0].y = static_cast<uint16_t*>(grad_x);
    v[0].numel = numel;
    v[0].group = nv ? fwd->group : 0;
    const float* am = nv ? d_group_amax : nullptr;
    return launch_format(f, 1, fwd->x_type, v, am, nullptr, n_groups, s);
}

const char* qf_status_string(qf_status s) {
    switch (s) {
        case QF_OK: return "QF_OK";
        case QF_ERR_INVALID_ARG: return "QF_ERR_INVALID_ARG: invalid argument";
        case QF_ERR_SHAPE: return "QF_ERR_SHAPE: invalid or unsupported shape";
        case QF_ERR_ALIGN: return "QF_ERR_ALIGN: pointer not 16-byte aligned";
        case QF_ERR_UNSUPPORTED: return "QF_ERR_UNSUPPORTED: unknown format or mode";
        case QF_ERR_CUDA: return "QF_ERR_CUDA: a CUDA call failed";
        case QF_ERR_TIMEOUT: return "QF_ERR_TIMEOUT: a bounded device wait gave up";
    }
    return "unknown qf_status";
}

const char* qf_last_error(void) { return g_err; }

int qf_version(void) { return (1 << 16) | 7; }

}  // extern "C"
