// cvt_probe.cu -- test probe: runs the library's own device conversion helpers
// (fp4_fake_quant_b200/csrc/qf_device.cuh) over every binary32 bit pattern of a
// range and records where the result changes, so a test can compare the hardware
// conversions with the oracle exhaustively.  Test infrastructure only.
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

}  // namespace

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
