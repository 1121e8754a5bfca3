// cvt_probe.cu -- test probe: runs the library's own device conversion helpers
// (fp4_fake_quant_b200/csrc/qf_device.cuh) over every binary32 bit pattern of a
// range and records where the result changes, so a test can compare the hardware
// conversions with the oracle exhaustively; and compares the library's two NVFP4
// block-scale derivations over every BF16 block amax.  Test infrastructure only.
#include <cstdint>
#include <cuda_runtime.h>

#include "qf_device.cuh"

namespace {

__device__ __forceinline__ uint32_t conv(int which, uint32_t u) {
    const float f = __uint_as_float(u);
    switch (which) {
        case 0: return qf::cvt_e2m1x2(0.0f, f) & 0xFu;            // E2M1, RNE, satfinite
        case 1: return qf::cvt_e4m3x2(0.0f, f) & 0xFFu;           // E4M3, RNE, satfinite
        case 2: return qf::cvt_bf16x2(0.0f, f) & 0xFFFFu;         // BF16, RNE
        default: return (uint32_t)__half_as_ushort(__float2half_rn(f));   // FP16, RNE
    }
}

__global__ void k_scan(int which, uint32_t lo, uint64_t n, uint32_t* pos, uint32_t* val,
                       uint32_t cap, unsigned long long* count) {
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const uint32_t u = lo + (uint32_t)i;
        const uint32_t r = conv(which, u);
        if (i == 0 || conv(which, u - 1u) != r) {
            const unsigned long long k = atomicAdd(count, 1ull);
            if (k < cap) { pos[k] = u; val[k] = r; }
        }
    }
}

__global__ void k_pairs(const float* a, const float* b, int n, uint32_t* e2m1, uint32_t* e4m3,
                        uint32_t* bf16) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        e2m1[i] = qf::cvt_e2m1x2(a[i], b[i]);
        e4m3[i] = qf::cvt_e4m3x2(a[i], b[i]);
        bf16[i] = qf::cvt_bf16x2(a[i], b[i]);
    }
}

__global__ void k_decode(uint32_t* e2m1_f16x2, uint32_t* e4m3_f16x2) {
    const uint32_t v = threadIdx.x;                     // 0..255
    e2m1_f16x2[v] = qf::cvt_e2m1x2_f16x2(v);
    e4m3_f16x2[v] = qf::cvt_e4m3x2_f16x2(v | (v << 8));
}

// 32-bit integer mixer (Wellons' "lowbias32"): pseudo-random test patterns
__device__ __forceinline__ uint32_t mix32(uint32_t x) {
    x ^= x >> 16;
    x *= 0x7feb352du;
    x ^= x >> 15;
    x *= 0x846ca68bu;
    x ^= x >> 16;
    return x;
}

// The NVFP4 block scale by the group tables (nv_block_scale_tab) against the division
// (nv_block_scale), bit for bit in (sb, S, 1/S): block y takes tensor scale s_t[y] and
// every non-negative BF16 block amax (0x0000..0x7FFF, +inf and NaNs included), then n_f32
// pseudo-random non-negative FP32 ones.  Counts the mismatches (the first 4 recorded as
// y, amax bits, sb by division, sb by table) and the blocks the table path decides itself.
__global__ void k_blockscale(const float* s_t, uint32_t n_f32, unsigned long long* bad,
                             uint32_t* first, unsigned long long* fast) {
    __shared__ qf::NvScaleTab tab;
    const float st = s_t[blockIdx.y];
    const float six = __fmul_rn(6.0f, st);
    const float yd = qf::nv_ratio_recip(six);
    if (yd != 0.0f) qf::nv_tab_fill(tab, st, threadIdx.x, blockDim.x);
    __syncthreads();
    const uint64_t total = 32768ull + n_f32;
    unsigned long long nfast = 0;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (uint64_t)gridDim.x * blockDim.x) {
        const uint32_t bits = i < 32768 ? (uint32_t)i << 16
                                        : mix32((uint32_t)i ^ (blockIdx.y * 0x9e3779b9u)) & 0x7FFFFFFFu;
        const float a = __uint_as_float(bits);
        uint32_t sb0, sb1;
        float S0, S1, inv0, inv1;
        qf::nv_block_scale(a, st, six, sb0, S0, inv0);
        qf::nv_block_scale_tab(a, st, six, yd, tab, sb1, S1, inv1);
        nfast += qf::nv_ratio_fast(__fmul_rn(a, yd), yd);
        if (sb0 != sb1 || __float_as_uint(S0) != __float_as_uint(S1) ||
            __float_as_uint(inv0) != __float_as_uint(inv1)) {
            const unsigned long long k = atomicAdd(bad, 1ull);
            if (k < 4) {
                first[4 * k] = blockIdx.y;
                first[4 * k + 1] = bits;
                first[4 * k + 2] = sb0;
                first[4 * k + 3] = sb1;
            }
        }
    }
    atomicAdd(fast + blockIdx.y, nfast);
}

// div_const(x, c, RN(1/c)) against __fdiv_rn(x, c) on every binary32 x (bit patterns
// lo .. lo + n - 1); counts mismatches (NaN results match any NaN) and records the first.
__global__ void k_divconst(float c, float c_inv, uint32_t lo, uint64_t n,
                           unsigned long long* bad, uint32_t* first) {
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const uint32_t u = lo + (uint32_t)i;
        const float x = __uint_as_float(u);
        const float a = qf::div_const(x, c, c_inv), b = __fdiv_rn(x, c);
        const bool same = __float_as_uint(a) == __float_as_uint(b) || (isnan(a) && isnan(b));
        if (!same && atomicAdd(bad, 1ull) == 0ull) *first = u;
    }
}

}  // namespace

extern "C" int probe_divconst(float c, float c_inv, uint32_t lo, uint64_t n,
                              unsigned long long* bad, uint32_t* first) {
    k_divconst<<<148 * 16, 256>>>(c, c_inv, lo, n, bad, first);
    return cudaDeviceSynchronize() == cudaSuccess ? 0 : 2;
}

extern "C" int probe_blockscale(const float* s_t, int n_st, uint32_t n_f32,
                                unsigned long long* bad, uint32_t* first,
                                unsigned long long* fast) {
    k_blockscale<<<dim3(64, (unsigned)n_st), 256>>>(s_t, n_f32, bad, first, fast);
    return cudaDeviceSynchronize() == cudaSuccess ? 0 : 2;
}

extern "C" int probe_scan(int which, uint32_t lo, uint32_t hi, uint32_t* pos, uint32_t* val,
                          uint32_t cap, unsigned long long* count) {
    if (hi < lo) return 1;
    const uint64_t n = (uint64_t)hi - lo + 1;
    k_scan<<<148 * 8, 256>>>(which, lo, n, pos, val, cap, count);
    return cudaDeviceSynchronize() == cudaSuccess ? 0 : 2;
}

extern "C" int probe_pairs(const float* a, const float* b, int n, uint32_t* e2m1, uint32_t* e4m3,
                           uint32_t* bf16) {
    k_pairs<<<(n + 255) / 256, 256>>>(a, b, n, e2m1, e4m3, bf16);
    return cudaDeviceSynchronize() == cudaSuccess ? 0 : 2;
}

extern "C" int probe_decode(uint32_t* e2m1_f16x2, uint32_t* e4m3_f16x2) {
    k_decode<<<1, 256>>>(e2m1_f16x2, e4m3_f16x2);
    return cudaDeviceSynchronize() == cudaSuccess ? 0 : 2;
}
