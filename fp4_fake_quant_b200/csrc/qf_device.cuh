// qf_device.cuh -- sm_100a kernels of the deployment-aligned simulated-quantization
// hot path (QATFactory project page: Method, "Framework overview" / "Numerics",
// "Supported formats" table).
//
// Design (HBM-bound streaming codec, no tensor cores):
//   * A call covers n tensors.  Their descriptors travel in a __grid_constant__
//     kernel parameter (no device allocation, no copy), each tensor split into
//     fixed-size "units" of elements; a unit is the work of one warp iteration.
//     A warp binary-searches the table for its first unit and walks forward.
//   * Inputs are BF16 or FP32 (latent master weights): every kernel is a template
//     on the element type XT and reads whole 16-byte vectors.
//   * MXFP4 (k_fp4): lane l holds 8 consecutive elements of each 256-element
//     sub-tile, so BF16 loads and stores are whole 512-byte warp transactions; the
//     4 lanes of a 32-element block reduce its max with shuffles.
//   * NVFP4 (k_nv): one lane per 16-element block, so the E4M3 block scale is
//     computed once per block and needs no shuffle.
//   * Q4_K (k_q4k): one lane per 32-element sub-block, four super-blocks per warp
//     iteration, BF16 traffic staged through padded shared-memory rows.
//   * Blackwell's native conversions do the format rounding:
//     cvt.rn.satfinite.e2m1x2.f32, cvt.rn.satfinite.e4m3x2.f32, cvt.rn.bf16x2.f32
//     and the reverse cvt.rn.f16x2.{e2m1x2,e4m3x2}.
//   * Every scale step is one IEEE binary32 operation with round-to-nearest-even
//     (__fdiv_rn, __frcp_rn, __fmul_rn, __fadd_rn); the library is built without
//     FMA contraction so the rounding order is the one the header documents (the
//     one explicit FMA, in the Q4_K dequant, is exact by construction).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

// Build-time launch-shape knobs, per kernel (the defaults are the shipped configuration,
// chosen by measurement on B200).  *_WAVES is the grid size in units of "one CTA per
// resident slot": 1 is a persistent grid, a large value one CTA per chunk of work.
#ifndef QF_MX_THREADS
#define QF_MX_THREADS 256
#endif
#ifndef QF_MX_WAVES
#define QF_MX_WAVES 1000
#endif
#ifndef QF_MX_PREFETCH
#define QF_MX_PREFETCH 0
#endif
#ifndef QF_NVB_THREADS
#define QF_NVB_THREADS 128      // NVFP4 fused pass, one lane per block (k_nv)
#endif
#ifndef QF_NVB_WAVES
#define QF_NVB_WAVES 1000
#endif
#ifndef QF_NVB_PREFETCH
#define QF_NVB_PREFETCH 0
#endif
#ifndef QF_NVB_U
#define QF_NVB_U 4              // 512-element sub-tiles per warp unit
#endif
#ifndef QF_FP4_U
#define QF_FP4_U 4              // 256-element sub-tiles per k_fp4 warp unit
#endif
#ifndef QF_FP4_LD
#define QF_FP4_LD 1             // load policy, see ld_stream
#endif
#ifndef QF_Q4K_THREADS
#define QF_Q4K_THREADS 512
#endif
#ifndef QF_Q4K_F32_THREADS
#define QF_Q4K_F32_THREADS 128  // the same for FP32 input (its lanes read their sub-blocks directly)
#endif
#ifndef QF_Q4K_WAVES
#define QF_Q4K_WAVES 1
#endif
#ifndef QF_Q4K_MSE_HOIST
#define QF_Q4K_MSE_HOIST 1      // MSE search: x + min_j formed once per sub-block, not per trial
#endif
#ifndef QF_Q4K_MSE_THREADS
#define QF_Q4K_MSE_THREADS QF_Q4K_THREADS
#endif
#ifndef QF_Q4K_PREFETCH
#define QF_Q4K_PREFETCH 0       // 1: register prefetch of each warp's next unit (BF16 input)
#endif
#ifndef QF_Q4K_LD
#define QF_Q4K_LD 1             // BF16 input: load form (ld_stream)
#endif
#ifndef QF_Q4K_MINB
#define QF_Q4K_MINB 0           // > 0: minimum resident CTAs per SM asked of the register allocator
#endif
#if QF_Q4K_MINB > 0
#define QF_Q4K_BOUNDS(t) __launch_bounds__(t, QF_Q4K_MINB)
#else
#define QF_Q4K_BOUNDS(t) __launch_bounds__(t)
#endif
#ifndef QF_AMAX_THREADS
#define QF_AMAX_THREADS 256
#endif
#ifndef QF_AMAX_WAVES
#define QF_AMAX_WAVES 1000
#endif
#ifndef QF_AMAX_LD
#define QF_AMAX_LD 2            // amax pass: load form (ld_stream; 2 measured best)
#endif
#ifndef QF_COPY_LD
#define QF_COPY_LD 1            // STE identity copy: load form (ld_stream; 1 measured best)
#endif
#ifndef QF_AMAX_ORDER
#define QF_AMAX_ORDER 0         // 0: one contiguous unit range per CTA, 1: grid-stride sweep
#endif
#ifndef QF_ST_POLICY
#define QF_ST_POLICY 0          // 0: default write-back stores, 1: streaming (.cs) stores
#endif

namespace qf {

constexpr int kThreads = 256;          // CTA size of the small helper kernels
constexpr unsigned kFull = 0xFFFFFFFFu;

// One tensor of a launch.
struct DevTensor {
    const void* x;          // input: BF16 or FP32 (the launch's element type)
    uint16_t* y;            // BF16 dequant out / STE grad_x (nullable)
    uint8_t* codes;         // packed nibbles / Q4_K blocks (nullable)
    uint8_t* scales;        // E4M3 / E8M0 bytes (nullable)
    const uint16_t* g;      // STE: upstream gradient
    int64_t numel;
    int64_t unit_begin;     // first global unit of this tensor
    int64_t unit_end;       // one past its last unit
    int32_t group;          // NVFP4 tie group
    int32_t pad;
};

template <int MAXT>
struct Table {
    DevTensor t[MAXT];
    int64_t total_units;
    const float* group_amax;    // NVFP4 tie-group amax (read) / qf_amax_tied output
    float* group_scale_out;     // NVFP4 s_t per group (nullable)
    float* tracked;             // qf_amax_tied running amax (nullable)
    int32_t n;
    int32_t n_groups;
    int32_t reverse;            // k_nv: visit the units from the last one down (see there)
};

// ------------------------------------------------------------------ PTX helpers
// Two FP32 -> one byte of two E2M1 codes: `hi` in bits 4-7, `lo` in bits 0-3.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float hi, float lo) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
// One byte of two E2M1 codes -> f16x2 (bits 4-7 -> upper half).
__device__ __forceinline__ uint32_t cvt_e2m1x2_f16x2(uint32_t b) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(r) : "r"(b));
    return r;
}
// Two FP32 -> two E4M3 bytes (hi in bits 8-15), round to nearest even, saturating.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float hi, float lo) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t cvt_e4m3x2_f16x2(uint32_t v) {
    uint32_t r;
    uint16_t h = (uint16_t)v;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(h));
    return r;
}
// Two FP32 -> BF16x2 (hi in the upper half), round to nearest even.
__device__ __forceinline__ uint32_t cvt_bf16x2(float hi, float lo) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float f16_lo(uint32_t h2) {
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}
__device__ __forceinline__ float f16_hi(uint32_t h2) {
    return __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
}
// Paired FP32 arithmetic of sm_100 (two independent lanes per instruction); each
// half rounds exactly as the scalar mul.rn / add.rn / fma.rn.f32 of the same
// operands.  One rule on their use: a paired product must not feed an add.  The
// code generator was seen to fuse a paired multiply and a following paired add
// into one rounding despite the explicit .rn (and also when the product was
// written as fma(a, b, -0)); a parity test caught it.  So paired products here
// feed only conversions, comparisons and selects, paired adds take no product,
// and every product that is added to something is a scalar __fmul_rn.
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
// Asynchronous 8-byte copy global -> shared; src_bytes = 0 writes zeros and
// reads nothing.  A thread's copies complete in commit-group order; cp_async_wait<N>
// blocks in hardware until at most N of the thread's groups are pending.
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
    return v;
}
// L2 prefetch of the line holding p; nothing waits for it
__device__ __forceinline__ void prefetch_line_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 16-byte streaming load on the read-only path.  LD = 0: no L1 allocation and a
// 256-byte L2 prefetch; 1: plain non-coherent load; 2: no L1 allocation; 3: ordinary
// (coherent) load, for a kernel that writes the buffer it reads (an in-place pass:
// the .nc forms require the data to stay unwritten for the kernel's lifetime).
template <int LD = 0>
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 v;
    if (LD == 0)
        asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
            : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    else if (LD == 1)
        asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
            : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    else if (LD == 2)
        asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
            : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));

    else
        asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_v4(void* p, uint4 v) {
#if QF_ST_POLICY == 1
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w) : "memory");
#else
    *reinterpret_cast<uint4*>(p) = v;
#endif
}

// bf16x2 helpers on raw bits
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&a),
                               *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t bmin2(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmin2(*reinterpret_cast<__nv_bfloat162*>(&a),
                               *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

// ------------------------------------------------------------------ element chunks
// N consecutive input elements of type XT (uint16_t = BF16 bits, float = FP32) held
// in registers as whole 16-byte vectors.
template <typename XT, int N>
struct Elems {
    static constexpr bool kBf16 = sizeof(XT) == 2;
    static constexpr int kVec = N * (int)sizeof(XT) / 16;
    uint4 v[kVec];

    __device__ __forceinline__ uint32_t word(int i) const {
        const uint4& q = v[i >> 2];
        const int k = i & 3;
        return k == 0 ? q.x : k == 1 ? q.y : k == 2 ? q.z : q.w;
    }
    // element k as FP32 (exact)
    __device__ __forceinline__ float get(int k) const {
        if constexpr (kBf16) return (k & 1) ? bf16_hi(word(k >> 1)) : bf16_lo(word(k >> 1));
        else return __uint_as_float(word(k));
    }
    // FP32 bit pattern of max |x| (non-negative floats order like their bit patterns)
    __device__ __forceinline__ uint32_t amax_bits() const {
        if constexpr (kBf16) {
            uint32_t m = word(0) & 0x7FFF7FFFu;
#pragma unroll
            for (int i = 1; i < 4 * kVec; ++i) m = bmax2(m, word(i) & 0x7FFF7FFFu);
            return max(m & 0xFFFFu, m >> 16) << 16;
        } else {
            uint32_t m = word(0) & 0x7FFFFFFFu;
#pragma unroll
            for (int i = 1; i < 4 * kVec; ++i) m = max(m, word(i) & 0x7FFFFFFFu);
            return m;
        }
    }
    // min and max of the elements
    __device__ __forceinline__ void minmax(float& lo, float& hi) const {
        if constexpr (kBf16) {
            uint32_t mx = word(0), mn = word(0);
#pragma unroll
            for (int i = 1; i < 4 * kVec; ++i) { mx = bmax2(mx, word(i)); mn = bmin2(mn, word(i)); }
            hi = fmaxf(bf16_lo(mx), bf16_hi(mx));
            lo = fminf(bf16_lo(mn), bf16_hi(mn));
        } else {
            hi = get(0);
            lo = hi;
#pragma unroll
            for (int k = 1; k < N; ++k) { hi = fmaxf(hi, get(k)); lo = fminf(lo, get(k)); }
        }
    }
    template <int LD>
    __device__ __forceinline__ void load(const XT* p, bool ok) {
#pragma unroll
        for (int i = 0; i < kVec; ++i)
            v[i] = ok ? ld_stream<LD>(reinterpret_cast<const uint8_t*>(p) + 16 * i)
                      : make_uint4(0, 0, 0, 0);
    }
};

// The tensor that owns unit u, by binary search over the units' first indices
// (for a warp's first unit).
template <int MAXT>
__device__ __forceinline__ int locate_tensor(const Table<MAXT>& P, int64_t u) {
    int lo = 0, hi = P.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.t[mid].unit_begin <= u) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Walk the descriptor table forward to the tensor that owns unit u (a warp visits
// its units in increasing order, so after locate_tensor this is amortised O(1)).
template <int MAXT>
__device__ __forceinline__ int find_tensor(const Table<MAXT>& P, int ti, int64_t u) {
    while (u >= P.t[ti].unit_end) ++ti;
    return ti;
}

// NVFP4 tensor scale of a tie group: s_t = amax_g / (6 * 448).
__device__ __forceinline__ float nv_tensor_scale(float amax_g) { return __fdiv_rn(amax_g, 2688.0f); }

// NVFP4 block scale from the block amax: sb = E4M3(amax_b / (6 s_t)), S = f32(sb) s_t,
// inv = 1/S (0 when S == 0; sb = 0 when s_t == 0).
__device__ __forceinline__ void nv_block_scale(float amax_b, float s_t, float six_st,
                                               uint32_t& sb, float& S, float& inv) {
    sb = 0;
    S = 0.0f;
    inv = 0.0f;
    if (s_t != 0.0f) {
        const float ratio = __fdiv_rn(amax_b, six_st);
        sb = cvt_e4m3x2(0.0f, ratio) & 0xFFu;
        S = __fmul_rn(f16_lo(cvt_e4m3x2_f16x2(sb)), s_t);
        inv = (S == 0.0f) ? 0.0f : __frcp_rn(S);
    }
}

// NVFP4 block scale from a tie group's tables.  The divisor 6 s_t of the block ratio is
// one number per tie group, so its reciprocal yd = RN(1 / (6 s_t)) is taken once, and
// q0 = RN(amax_b * yd) lies within two FP32 steps of the ratio RN(amax_b / (6 s_t))
// wherever both fall in one binade (the product's relative error is below 2^-24, and
// each rounding adds at most half a step).  The block byte is the ratio rounded to E4M3;
// in E4M3's normal range [2^-6, 448] every rounding boundary has the low 20 mantissa bits
// 0x80000, so where q0's low bits are more than 3 steps from that pattern, q0 and the
// ratio round to the same byte, and below 2^-11 (or above 2^9) both give 0 (or the
// saturated 448).  Everything else (near a boundary, E4M3's subnormal range, a NaN, or a
// group whose 6 s_t lies outside [2^-80, 2^100], marked by yd = 0) takes the division of
// nv_block_scale.  S and 1/S come from the group's table of the 128 E4M3 bytes, filled
// with nv_block_scale's own operations.
struct NvScaleTab {
    float S[128];
    float inv[128];
};
// entries i, i + n, ... of the table of tensor scale s_t (s_t != 0)
__device__ __forceinline__ void nv_tab_fill(NvScaleTab& t, float s_t, int i, int n) {
    for (int c = i; c < 128; c += n) {
        const float S = __fmul_rn(f16_lo(cvt_e4m3x2_f16x2((uint32_t)c)), s_t);
        t.S[c] = S;
        t.inv[c] = S == 0.0f ? 0.0f : __frcp_rn(S);
    }
}
// yd for a group, 0 where the division is always taken
__device__ __forceinline__ float nv_ratio_recip(float six_st) {
    return (six_st >= 0x1p-80f && six_st <= 0x1p100f) ? __frcp_rn(six_st) : 0.0f;
}
// whether q0 = RN(amax_b * yd) rounds to the block byte itself
__device__ __forceinline__ bool nv_ratio_fast(float q0, float yd) {
    const uint32_t low = __float_as_uint(q0) & 0xFFFFFu;
    return yd != 0.0f && (q0 < 0x1p-11f || q0 > 0x1p9f || (q0 >= 0x1p-6f && low - 0x7FFFDu > 6u));
}
__device__ __forceinline__ void nv_block_scale_tab(float amax_b, float s_t, float six_st, float yd,
                                                   const NvScaleTab& t, uint32_t& sb, float& S,
                                                   float& inv) {
    const float q0 = __fmul_rn(amax_b, yd);
    if (__builtin_expect(nv_ratio_fast(q0, yd), 1)) {
        sb = cvt_e4m3x2(0.0f, q0) & 0xFFu;
        S = t.S[sb];
        inv = t.inv[sb];
    } else {
        nv_block_scale(amax_b, s_t, six_st, sb, S, inv);
    }
}

// ------------------------------------------------------------------ k_fp4 (MXFP4; STE)
// Per-lane result of the FP4 codec for 8 elements.
struct Fp4Lane {
    uint32_t codes;     // 8 nibbles, element k in bits 4k..4k+3
    uint32_t scale;     // block scale byte
    uint4 y;            // 8 BF16
    float q[8];         // scaled values (for the clipped STE)
};

// TAB (NVFP4): the block scale from the group's tables (nv_block_scale_tab; yd, tab given).
template <bool NV, bool WANT_Y, bool TAB = false, typename XT>
__device__ __forceinline__ void fp4_lane(const Elems<XT, 8>& x, float s_t, float six_st,
                                         Fp4Lane& o, float yd = 0.0f,
                                         const NvScaleTab* tab = nullptr) {
    uint32_t a = x.amax_bits();
    a = max(a, __shfl_xor_sync(kFull, a, 1));
    if (!NV) a = max(a, __shfl_xor_sync(kFull, a, 2));
    float S, inv;
    if (NV) {
        uint32_t sb;
        if constexpr (TAB) nv_block_scale_tab(__uint_as_float(a), s_t, six_st, yd, *tab, sb, S, inv);
        else nv_block_scale(__uint_as_float(a), s_t, six_st, sb, S, inv);
        o.scale = sb;
    } else {
        // E8M0: e = floor(log2 amax) - 2 clamped to >= -127; byte = e + 127 = max(E - 2, 0)
        const uint32_t E = a >> 23;
        const uint32_t c = E > 2u ? E - 2u : 0u;
        o.scale = c;
        inv = __uint_as_float((254u - c) << 23);                          // 2^-e
        S = c ? __uint_as_float(c << 23) : __uint_as_float(0x00400000u);  // 2^e (2^-127: subnormal)
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) o.q[k] = __fmul_rn(x.get(k), inv);
    if (NV && __builtin_expect(isinf(inv), 0)) {
        // 1/S overflowed (S < 2^-128): a zero keeps its own sign instead of 0 * inf
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (x.get(k) == 0.0f) o.q[k] = x.get(k);
    }
    uint32_t b[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) b[k] = cvt_e2m1x2(o.q[2 * k + 1], o.q[2 * k]);
    o.codes = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    if (WANT_Y) {
        uint32_t yw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t h2 = cvt_e2m1x2_f16x2(b[k]);
            yw[k] = cvt_bf16x2(__fmul_rn(f16_hi(h2), S), __fmul_rn(f16_lo(h2), S));
        }
        o.y = make_uint4(yw[0], yw[1], yw[2], yw[3]);
    }
}

template <typename XT, int U, int MODE>
struct UnitLoad {
    Elems<XT, 8> v[U];
    uint4 gv[MODE == 1 ? U : 1];
};

template <typename XT, int U, int MODE>
__device__ __forceinline__ void load_unit(const DevTensor& T, int64_t e0, int lane,
                                          UnitLoad<XT, U, MODE>& L) {
    const XT* x = static_cast<const XT*>(T.x);
#pragma unroll
    for (int s = 0; s < U; ++s) {
        const int64_t e = e0 + s * 256 + lane * 8;
        const bool ok = e < T.numel;
        L.v[s].template load<QF_FP4_LD>(x + e, ok);
        // coherent: grad_x may be grad_y (each element is read before its thread writes it)
        if (MODE == 1) L.gv[s] = ok ? ld_stream<3>(T.g + e) : make_uint4(0, 0, 0, 0);
    }
}

// MXFP4 fused fake-quant + pack (MODE 0), or the MXFP4 clipped STE (MODE 1); the
// library launches it with NV = false (NVFP4 has the lane-per-block k_nv / k_nv_ste,
// and the NV = true form is kept as the same kernel's 8-element-lane variant).
// A unit is U sub-tiles of 256 elements.
template <bool NV, typename XT, int U, int MAXT, int MODE, int THREADS, int PREFETCH>
__global__ void __launch_bounds__(THREADS) k_fp4(const __grid_constant__ Table<MAXT> P) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * THREADS + threadIdx.x) >> 5;
    const int64_t nwarps = (int64_t(gridDim.x) * THREADS) >> 5;
    constexpr int kUnit = 256 * U;
    if (NV && MODE == 0 && blockIdx.x == 0 && P.group_scale_out) {
        for (int g = threadIdx.x; g < P.n_groups; g += THREADS)
            P.group_scale_out[g] = nv_tensor_scale(P.group_amax[g]);
    }
    int64_t u = warp;
    if (u >= P.total_units) return;
    int ti = locate_tensor(P, u);
    UnitLoad<XT, U, MODE> cur;
    load_unit<XT, U, MODE>(P.t[ti], (u - P.t[ti].unit_begin) * kUnit, lane, cur);
    int cur_t = -1;
    float s_t = 0.0f, six_st = 0.0f;
    while (true) {
        const int64_t un = u + nwarps;
        int tn = ti;
        UnitLoad<XT, U, MODE> nxt;
        if (PREFETCH && un < P.total_units) {
            tn = find_tensor(P, ti, un);
            load_unit<XT, U, MODE>(P.t[tn], (un - P.t[tn].unit_begin) * kUnit, lane, nxt);
        }
        const DevTensor& T = P.t[ti];
        if (NV && ti != cur_t) {
            s_t = nv_tensor_scale(P.group_amax[T.group]);
            six_st = __fmul_rn(6.0f, s_t);
            cur_t = ti;
        }
        const int64_t e0 = (u - T.unit_begin) * kUnit;
#pragma unroll
        for (int s = 0; s < U; ++s) {
            const int64_t e = e0 + s * 256 + lane * 8;
            const bool ok = e < T.numel;
            Fp4Lane o;
            if (MODE == 0) {
                if (T.y) fp4_lane<NV, true>(cur.v[s], s_t, six_st, o);
                else fp4_lane<NV, false>(cur.v[s], s_t, six_st, o);
                if (ok) {
                    if (T.y) st_v4(T.y + e, o.y);
                    if (T.codes) *reinterpret_cast<uint32_t*>(T.codes + (e >> 1)) = o.codes;
                    if (T.scales && (lane & (NV ? 1 : 3)) == 0)
                        T.scales[e >> (NV ? 4 : 5)] = (uint8_t)o.scale;
                }
            } else {
                fp4_lane<NV, false>(cur.v[s], s_t, six_st, o);
                if (ok) {
                    const uint32_t gw[4] = {cur.gv[s].x, cur.gv[s].y, cur.gv[s].z, cur.gv[s].w};
                    uint32_t r[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint32_t lo = fabsf(o.q[2 * k]) <= 6.0f ? (gw[k] & 0xFFFFu) : 0u;
                        uint32_t hi = fabsf(o.q[2 * k + 1]) <= 6.0f ? (gw[k] & 0xFFFF0000u) : 0u;
                        r[k] = lo | hi;
                    }
                    st_v4(T.y + e, make_uint4(r[0], r[1], r[2], r[3]));
                }
            }
        }
        if (un >= P.total_units) break;
        u = un;
        if (PREFETCH) {
            ti = tn;
            cur = nxt;
        } else {
            ti = find_tensor(P, ti, u);
            load_unit<XT, U, MODE>(P.t[ti], (u - P.t[ti].unit_begin) * kUnit, lane, cur);
        }
    }
}

// ------------------------------------------------------------------ NVFP4, lane per block
// NVFP4 fake-quant + pack with one lane per 16-element block: a warp sub-tile is 32
// consecutive blocks (512 elements) and lane l owns block l, so the E4M3 block scale
// (one IEEE divide, one reciprocal) is computed once per block and the block max
// needs no shuffle.  A lane reads its block with consecutive 16-byte loads (together
// they cover whole sectors; the later ones are served from L1) and writes 32 bytes
// of BF16, 8 bytes of codes and 1 scale byte: the warp's code and scale stores are
// contiguous 256- and 32-byte runs.
template <typename XT, int U, int LD>
__device__ __forceinline__ void nv_load_unit(const DevTensor& T, int64_t e0, int lane,
                                             Elems<XT, 16> (&v)[U]) {
    const XT* x = static_cast<const XT*>(T.x);
#pragma unroll
    for (int s = 0; s < U; ++s) {
        const int64_t e = e0 + s * 512 + lane * 16;
        v[s].template load<LD>(x + e, e < T.numel);
    }
}

// Encode one warp unit (U sub-tiles of 512 elements starting at element e0).
template <typename XT, int U>
__device__ __forceinline__ void nv_encode_unit(const DevTensor& T, int64_t e0, int lane,
                                               const Elems<XT, 16> (&cur)[U], float s_t,
                                               float six_st) {
#pragma unroll
    for (int s = 0; s < U; ++s) {
        const int64_t e = e0 + s * 512 + lane * 16;
        const Elems<XT, 16>& x = cur[s];
        uint32_t sb;
        float S, inv;
        nv_block_scale(__uint_as_float(x.amax_bits()), s_t, six_st, sb, S, inv);
        float q[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) q[k] = __fmul_rn(x.get(k), inv);
        if (__builtin_expect(isinf(inv), 0)) {
            // 1/S overflowed (S < 2^-128): a zero keeps its own sign instead of 0 * inf
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if (x.get(k) == 0.0f) q[k] = x.get(k);
        }
        uint32_t b[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) b[k] = cvt_e2m1x2(q[2 * k + 1], q[2 * k]);
        if (e < T.numel) {
            if (T.y) {
                uint32_t yw[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t h2 = cvt_e2m1x2_f16x2(b[k]);
                    yw[k] = cvt_bf16x2(__fmul_rn(f16_hi(h2), S), __fmul_rn(f16_lo(h2), S));
                }
                st_v4(T.y + e, make_uint4(yw[0], yw[1], yw[2], yw[3]));
                st_v4(T.y + e + 8, make_uint4(yw[4], yw[5], yw[6], yw[7]));
            }
            if (T.codes) {
                const uint32_t lo = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
                const uint32_t hi = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
                *reinterpret_cast<uint2*>(T.codes + (e >> 1)) = make_uint2(lo, hi);
            }
            if (T.scales) T.scales[e >> 4] = (uint8_t)sb;
        }
    }
}

// DEP_AMAX: launched as a programmatic dependent of the amax kernel that produces
// P.group_amax (and writes nothing this kernel reads otherwise).  The first unit of
// x is loaded before griddepcontrol.wait -- x was final before the amax kernel
// started -- and the group amax is read only after it, so the loads of this grid's
// first wave overlap the end of the amax grid.
//
// P.reverse: the warps take the units from the last one down.  A pass that follows one
// over the same data (the tie-group amax, or the merge that wrote x) ends with its last
// units' lines in L2, so the first units this grid reads come from L2, and lines it
// overwrites in place need not be written back first.  The results do not depend on the
// order.
template <typename XT, int U, int MAXT, int THREADS, int PREFETCH, int LD = QF_FP4_LD,
          bool DEP_AMAX = false>
__global__ void __launch_bounds__(THREADS) k_nv(const __grid_constant__ Table<MAXT> P) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * THREADS + threadIdx.x) >> 5;
    const int64_t nwarps = (int64_t(gridDim.x) * THREADS) >> 5;
    constexpr int kUnit = 512 * U;
    const bool rev = P.reverse != 0;
    // the unit a warp's logical index stands for, and the tensor that owns it
    auto phys = [&](int64_t lu) { return rev ? P.total_units - 1 - lu : lu; };
    auto owner = [&](int hint, int64_t pu) { return rev ? locate_tensor(P, pu) : find_tensor(P, hint, pu); };
    int64_t u = warp;
    int ti = 0;
    Elems<XT, 16> cur[U], nxt[U];
    if (u < P.total_units) {
        ti = locate_tensor(P, phys(u));
        nv_load_unit<XT, U, LD>(P.t[ti], (phys(u) - P.t[ti].unit_begin) * kUnit, lane, cur);
    }
    if (DEP_AMAX) asm volatile("griddepcontrol.wait;" ::: "memory");
    if (blockIdx.x == 0 && P.group_scale_out) {
        for (int g = threadIdx.x; g < P.n_groups; g += THREADS)
            P.group_scale_out[g] = nv_tensor_scale(P.group_amax[g]);
    }
    if (u >= P.total_units) return;
    int cur_t = -1;
    float s_t = 0.0f, six_st = 0.0f;
    while (true) {
        const int64_t un = u + nwarps;
        int tn = ti;
        if (PREFETCH && un < P.total_units) {
            tn = owner(ti, phys(un));
            nv_load_unit<XT, U, LD>(P.t[tn], (phys(un) - P.t[tn].unit_begin) * kUnit, lane, nxt);
        }
        const DevTensor& T = P.t[ti];
        if (ti != cur_t) {
            s_t = nv_tensor_scale(P.group_amax[T.group]);
            six_st = __fmul_rn(6.0f, s_t);
            cur_t = ti;
        }
        nv_encode_unit<XT, U>(T, (phys(u) - T.unit_begin) * kUnit, lane, cur, s_t, six_st);
        if (un >= P.total_units) break;
        u = un;
        if (PREFETCH) {
            ti = tn;
#pragma unroll
            for (int i = 0; i < U; ++i) cur[i] = nxt[i];
        } else {
            ti = owner(ti, phys(u));
            nv_load_unit<XT, U, LD>(P.t[ti], (phys(u) - P.t[ti].unit_begin) * kUnit, lane, cur);
        }
    }
}

// NVFP4 clipped STE with one lane per 16-element block (the k_nv layout): the lane
// derives its block's scale from x exactly as the forward pass does and keeps the
// gradient of every element with |x * (1/S)| <= 6 (a zero x counts as 0).  grad_y is
// read with ordinary loads: grad_x may be grad_y.
template <typename XT, int U, int MAXT, int THREADS>
__global__ void __launch_bounds__(THREADS) k_nv_ste(const __grid_constant__ Table<MAXT> P) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * THREADS + threadIdx.x) >> 5;
    const int64_t nwarps = (int64_t(gridDim.x) * THREADS) >> 5;
    constexpr int kUnit = 512 * U;
    if (warp >= P.total_units) return;
    int ti = locate_tensor(P, warp);
    int cur_t = -1;
    float s_t = 0.0f, six_st = 0.0f;
    for (int64_t u = warp; u < P.total_units; u += nwarps) {
        ti = find_tensor(P, ti, u);
        const DevTensor& T = P.t[ti];
        if (ti != cur_t) {
            s_t = nv_tensor_scale(P.group_amax[T.group]);
            six_st = __fmul_rn(6.0f, s_t);
            cur_t = ti;
        }
        const int64_t e0 = (u - T.unit_begin) * kUnit;
        Elems<XT, 16> x[U];
        nv_load_unit<XT, U, QF_FP4_LD>(T, e0, lane, x);
        uint4 g[U][2];
#pragma unroll
        for (int s = 0; s < U; ++s) {
            const int64_t e = e0 + s * 512 + lane * 16;
            const bool ok = e < T.numel;
            g[s][0] = ok ? ld_stream<3>(T.g + e) : make_uint4(0, 0, 0, 0);
            g[s][1] = ok ? ld_stream<3>(T.g + e + 8) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int s = 0; s < U; ++s) {
            const int64_t e = e0 + s * 512 + lane * 16;
            uint32_t sb;
            float S, inv;
            nv_block_scale(__uint_as_float(x[s].amax_bits()), s_t, six_st, sb, S, inv);
            const bool inf_inv = isinf(inv);
            uint32_t keep = 0;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                float q = __fmul_rn(x[s].get(k), inv);
                if (inf_inv && x[s].get(k) == 0.0f) q = x[s].get(k);
                keep |= (uint32_t)(fabsf(q) <= 6.0f) << k;
            }
            uint32_t w[8] = {g[s][0].x, g[s][0].y, g[s][0].z, g[s][0].w,
                             g[s][1].x, g[s][1].y, g[s][1].z, g[s][1].w};
#pragma unroll
            for (int k = 0; k < 8; ++k)
                w[k] = (((keep >> (2 * k)) & 1u) ? (w[k] & 0xFFFFu) : 0u) |
                       (((keep >> (2 * k + 1)) & 1u) ? (w[k] & 0xFFFF0000u) : 0u);
            if (e < T.numel) {
                st_v4(T.y + e, make_uint4(w[0], w[1], w[2], w[3]));
                st_v4(T.y + e + 8, make_uint4(w[4], w[5], w[6], w[7]));
            }
        }
    }
}

// RN(x / c) for a constant divisor c > 0, given c_inv = RN(1 / c): q0 = RN(x * c_inv)
// and one correction by the exact residual x - q0 c (Markstein's correction step, as in
// P. Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990); a zero residual keeps q0 (and the sign of a
// zero quotient).  Magnitudes outside [2^-100, 2^100], and NaN, take the division itself.
// For each constant the kernels use, a GPU test compares it with the IEEE division on
// every one of the 2^32 inputs.
__device__ __forceinline__ float div_const(float x, float c, float c_inv) {
    const float ax = fabsf(x);
    if (__builtin_expect(ax <= 0x1p100f && (ax >= 0x1p-100f || ax == 0.0f), 1)) {
        const float q0 = __fmul_rn(x, c_inv);
        const float r = __fmaf_rn(-q0, c, x);
        return r == 0.0f ? q0 : __fmaf_rn(r, c_inv, q0);
    }
    return __fdiv_rn(x, c);
}
#ifndef QF_DIVCONST
#define QF_DIVCONST 1           // Q4_K fits: divisions by constants through div_const
#endif
// x / c for one of the Q4_K fits' constant divisors (c_inv = RN(1 / c))
__device__ __forceinline__ float q4k_div(float x, float c, float c_inv) {
    return QF_DIVCONST ? div_const(x, c, c_inv) : __fdiv_rn(x, c);
}

// ------------------------------------------------------------------ Q4_K
// One lane per 32-element sub-block: a warp iteration covers 4 super-blocks (1024
// elements) and lane l owns sub-block j = l / 4 of super-block b = l % 4, so the
// per-sub-block and per-super-block scalar work (divides, FP16 and integer
// conversions) is amortised over 32 elements.  BF16 traffic stays fully coalesced:
// the warp stages its 2 KB through shared memory (one 528-byte row per
// super-block, 16 bytes of padding so that the lanes' 16-byte accesses hit
// distinct banks) and transposes there.  FP32 input is read by each lane directly
// (its 128-byte sub-block, whole lines, the later vectors served from L1).
constexpr int kQ4kRow = 528;
constexpr int kQ4kWarpBytes = 4 * kQ4kRow;
constexpr float kRound = 12582912.0f;      // 1.5 * 2^23: v + kRound rounds v to an integer (RNE)

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z),
                 "=r"(v.w) : "r"(addr) : "memory");
    return v;
}

// Squared dequantization error of one sub-block at two trial scales (offset min_j),
// summed in element order: q = clamp(RNE((x + min_j) / scale), 0, 15),
// err = sum (x - (scale*q - min_j))^2, one rounding per operation.  The two trials
// share sm_100's paired FP32 pipe where no product feeds an add (the scaled value
// and the rounding to an integer); the products scale*q and r*r, which are added
// to, stay scalar.  The error is accumulated as (dq - x)^2, whose square equals
// that of x - dq bit for bit (round-to-nearest is symmetric, so dq - x is exactly
// -(x - dq)).  x + min_j >= +0 always (min_j >= -min x), so with a finite reciprocal
// the scaled value is >= +0 and only the upper clamp can act: LOWER = false drops the
// lower one.  LOWER = true keeps it for a reciprocal that overflowed (0 * inf).
// XM: the sub-block's x + min_j, formed once for all trials (QF_Q4K_MSE_HOIST), or NULL.
template <typename XT, bool LOWER>
__device__ __forceinline__ float2 q4k_sub_err2(const Elems<XT, 32>& x, float2 scale, float min_j,
                                               const float* XM) {
    const float2 inv = make_float2(__frcp_rn(scale.x), __frcp_rn(scale.y));
    const float2 rnd = make_float2(kRound, kRound), nrnd = make_float2(-kRound, -kRound);
    float2 err = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const float xk = x.get(k);
        const float xm = QF_Q4K_MSE_HOIST ? XM[k] : __fadd_rn(xk, min_j);
        const float2 t = mul2_rn(make_float2(xm, xm), inv);
        const float2 c = LOWER ? make_float2(fminf(fmaxf(t.x, 0.0f), 15.0f), fminf(fmaxf(t.y, 0.0f), 15.0f))
                               : make_float2(fminf(t.x, 15.0f), fminf(t.y, 15.0f));
        const float2 q = add2_rn(add2_rn(c, rnd), nrnd);
        const float2 dq = make_float2(__fsub_rn(__fmul_rn(scale.x, q.x), min_j),
                                      __fsub_rn(__fmul_rn(scale.y, q.y), min_j));
        const float2 r = add2_rn(dq, make_float2(-xk, -xk));
        err = make_float2(__fadd_rn(err.x, __fmul_rn(r.x, r.x)),
                          __fadd_rn(err.y, __fmul_rn(r.y, r.y)));
    }
    return err;
}
// MSE-searched sub-block scale: with the offset fixed, try scale = (hi + min_j) / n
// for n = 15 (the min/max fit) and then 14, 14.5, 15.5, 16, 16.5, 17, 17.5, 18; keep
// the least squared error (a later trial must be strictly smaller).  The errors are
// computed two trials at a time and then compared in trial order.
template <typename XT, bool LOWER>
__device__ __forceinline__ float q4k_search_scale_t(const Elems<XT, 32>& x, float range,
                                                    float best, float s18, float min_j) {
    const float s14 = q4k_div(range, 14.0f, 1.0f / 14.0f);
    float xm[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) xm[k] = QF_Q4K_MSE_HOIST ? __fadd_rn(x.get(k), min_j) : 0.0f;
    const float2 e0 = q4k_sub_err2<XT, LOWER>(x, make_float2(best, s14), min_j, xm);
    float best_err = e0.x;
    if (e0.y < best_err) {
        best_err = e0.y;
        best = s14;
    }
    // the remaining trials in pairs (14.5, 15.5), (16, 16.5), (17, 17.5) and 18 alone
    // (its pair's second half repeats it and is ignored)
#pragma unroll 1
    for (int p = 0; p < 4; ++p) {
        const float na = p == 0 ? 14.5f : p == 1 ? 16.0f : p == 2 ? 17.0f : 18.0f;
        const float nb = p == 0 ? 15.5f : p == 1 ? 16.5f : p == 2 ? 17.5f : 18.0f;
        const float ia = p == 0 ? 1.0f / 14.5f : p == 1 ? 1.0f / 16.0f : p == 2 ? 1.0f / 17.0f
                                                                         : 1.0f / 18.0f;
        const float ib = p == 0 ? 1.0f / 15.5f : p == 1 ? 1.0f / 16.5f : p == 2 ? 1.0f / 17.5f
                                                                         : 1.0f / 18.0f;
        const float2 sc = make_float2(p == 3 ? s18 : q4k_div(range, na, ia), q4k_div(range, nb, ib));
        const float2 err = q4k_sub_err2<XT, LOWER>(x, sc, min_j, xm);
        if (err.x < best_err) {
            best_err = err.x;
            best = sc.x;
        }
        if (p < 3 && err.y < best_err) {
            best_err = err.y;
            best = sc.y;
        }
    }
    return best;
}
template <typename XT>
__device__ __forceinline__ float q4k_search_scale(const Elems<XT, 32>& x, float hi, float min_j) {
    const float range = __fadd_rn(hi, min_j);
    const float best = q4k_div(range, 15.0f, 1.0f / 15.0f);
    if (best == 0.0f) return best;
    // range / 18 is the smallest trial scale: when its reciprocal is finite, so are all
    const float s18 = q4k_div(range, 18.0f, 1.0f / 18.0f);
    if (__frcp_rn(s18) <= 3.402823466e38f)
        return q4k_search_scale_t<XT, false>(x, range, best, s18, min_j);
    return q4k_search_scale_t<XT, true>(x, range, best, s18, min_j);
}

// Per-lane fit of one sub-block; returns the super-block's FP16 d / dmin bits, this
// sub-block's 6-bit sc / m, its s = d*sc, mm = dmin*m and inv = 1/s.  MSE selects
// the searched sub-block scale instead of the min/max one.
struct Q4kFit { uint32_t dbits, dminbits, sc, m; float s, mm, inv; };

template <typename XT, bool MSE>
__device__ __forceinline__ Q4kFit q4k_fit(const Elems<XT, 32>& x) {
    float lo, hi;
    x.minmax(lo, hi);
    const float min_j = lo < 0.0f ? -lo : 0.0f;
    const float scale_j = MSE ? q4k_search_scale(x, hi, min_j)
                              : q4k_div(__fadd_rn(hi, min_j), 15.0f, 1.0f / 15.0f);
    float ms = scale_j, mm = min_j;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {               // the 8 lanes of this super-block
        ms = fmaxf(ms, __shfl_xor_sync(kFull, ms, o));
        mm = fmaxf(mm, __shfl_xor_sync(kFull, mm, o));
    }
    const __half dh = __float2half_rn(q4k_div(ms, 63.0f, 1.0f / 63.0f));
    const __half dmh = __float2half_rn(q4k_div(mm, 63.0f, 1.0f / 63.0f));
    const float d = __half2float(dh), dmin = __half2float(dmh);
    Q4kFit f;
    f.dbits = __half_as_ushort(dh);
    f.dminbits = __half_as_ushort(dmh);
    f.sc = d == 0.0f ? 0u : (uint32_t)min(__float2int_rn(__fdiv_rn(scale_j, d)), 63);
    f.m = dmin == 0.0f ? 0u : (uint32_t)min(__float2int_rn(__fdiv_rn(min_j, dmin)), 63);
    f.s = __fmul_rn(d, (float)f.sc);
    f.mm = __fmul_rn(dmin, (float)f.m);
    f.inv = f.s == 0.0f ? 0.0f : __frcp_rn(f.s);
    return f;
}

// Elements, BF16 output and the 144-byte blocks of one warp unit (MODE 0): lane
// (b, j) holds sub-block j of super-block b in x with its fit f; sm_lane / sm_mine
// are the warp's staging rows (coalesced and transposed views).
template <typename XT>
__device__ __forceinline__ void q4k_emit_unit(const DevTensor& T, int64_t e0, int nsb, int lane,
                                              const Elems<XT, 32>& x, const Q4kFit& f,
                                              uint32_t sm_lane, uint32_t sm_mine) {
    const int b = lane & 3, j = lane >> 2;
    const bool have = b < nsb;
    const int64_t sb = (e0 >> 8) + b;                    // this lane's super-block in the tensor
    // elements: q = clamp(RNE((x + mm) * inv), 0, 15); y = BF16(s*q - mm)
    uint32_t qw[8];                              // q of elements 4t..4t+3, one per byte
    uint32_t yw[16];
    // two elements per step on the paired FP32 pipe (no paired product feeds an
    // add: the scaled value goes through the clamp first)
    const float2 mm2 = make_float2(f.mm, f.mm), inv2 = make_float2(f.inv, f.inv);
    const float2 rnd2 = make_float2(kRound, kRound), nrnd2 = make_float2(-kRound, -kRound);
    const float2 s2 = make_float2(f.s, f.s), nmm2 = make_float2(-f.mm, -f.mm);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float2 t = mul2_rn(add2_rn(make_float2(x.get(2 * k), x.get(2 * k + 1)), mm2),
                                 inv2);
        const float2 r = add2_rn(make_float2(fminf(fmaxf(t.x, 0.0f), 15.0f),
                                             fminf(fmaxf(t.y, 0.0f), 15.0f)), rnd2);
        if (k & 1) qw[k >> 1] = __byte_perm(qw[k >> 1], __byte_perm(__float_as_uint(r.x),
                                            __float_as_uint(r.y), 0x0040), 0x5410);
        else qw[k >> 1] = __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x0040);
        // y = RN(s*q - mm): s = d*sc has at most 17 significant bits and q at most 4,
        // so s*q is exact and one fused multiply-add rounds exactly once, as the
        // separate multiply and subtract do
        const float2 yv = fma2_rn(s2, add2_rn(r, nrnd2), nmm2);
        yw[k] = cvt_bf16x2(yv.y, yv.x);
    }
    if (T.y) {
        // stage y back through this lane's own 64 bytes, then store coalesced
#pragma unroll
        for (int p = 0; p < 4; ++p)
            sts128(sm_mine + 16 * p, make_uint4(yw[4 * p], yw[4 * p + 1], yw[4 * p + 2],
                                                yw[4 * p + 3]));
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (k < nsb) st_v4(T.y + e0 + 256 * k + 8 * lane, lds128(sm_lane + k * kQ4kRow));
    }
    if (T.codes) {
        // codes: byte l of chunk c = q[2c][l] | q[2c+1][l] << 4; the even sub-block's
        // lane writes bytes 0-15 of the chunk, the odd one bytes 16-31 (partner = lane ^ 4)
        const bool odd = j & 1;
        uint32_t out[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const uint32_t recv = __shfl_xor_sync(kFull, odd ? qw[t] : qw[4 + t], 4);
            out[t] = odd ? (recv | (qw[4 + t] << 4)) : (qw[t] | (recv << 4));
        }
        uint8_t* blk = T.codes + sb * 144;
        if (have) st_v4(blk + 16 + 16 * j, make_uint4(out[0], out[1], out[2], out[3]));
        // header: d, dmin, then the 12 bytes of 6-bit scales and mins
        const uint32_t smv = f.sc | (f.m << 8);
        const uint32_t o4 = __shfl_xor_sync(kFull, smv, 16);      // sub-block j ^ 4
        const uint32_t scB = o4 & 0xFF, mB = o4 >> 8;
        const uint32_t pk = ((f.sc & 63) | ((scB >> 4) << 6)) |
                            (((f.m & 63) | ((mB >> 4) << 6)) << 8) |
                            (((scB & 15) | ((mB & 15) << 4)) << 16);
        const uint32_t p1 = __shfl_sync(kFull, pk, b + 4);
        const uint32_t p2 = __shfl_sync(kFull, pk, b + 8);
        const uint32_t p3 = __shfl_sync(kFull, pk, b + 12);
        if (j == 0 && have) {
            const uint32_t l1 = __byte_perm(pk, p1, 0x0040), h1 = __byte_perm(p2, p3, 0x0040);
            const uint32_t l2 = __byte_perm(pk, p1, 0x0051), h2 = __byte_perm(p2, p3, 0x0051);
            const uint32_t l3 = __byte_perm(pk, p1, 0x0062), h3 = __byte_perm(p2, p3, 0x0062);
            st_v4(blk, make_uint4(f.dbits | (f.dminbits << 16), __byte_perm(l1, h1, 0x5410),
                                  __byte_perm(l2, h2, 0x5410), __byte_perm(l3, h3, 0x5410)));
        }
    }
}

// MODE 0: dequant (y) and/or 144-byte blocks (codes).  MODE 1: clipped STE, y = grad_x.
template <typename XT, int MAXT, int MODE, int THREADS, bool MSE>
__global__ void QF_Q4K_BOUNDS(THREADS) k_q4k(const __grid_constant__ Table<MAXT> P) {
    __shared__ __align__(16) uint8_t stage[THREADS / 32][kQ4kWarpBytes];
    constexpr bool kBf16 = sizeof(XT) == 2;
    const int lane = threadIdx.x & 31;
    const int b = lane & 3, j = lane >> 2;              // super-block of 4, sub-block of 8
    const uint32_t sm = (uint32_t)__cvta_generic_to_shared(stage[threadIdx.x >> 5]);
    const uint32_t sm_lane = sm + 16u * lane;           // coalesced view: row k at + k*528
    const uint32_t sm_mine = sm + b * kQ4kRow + 64u * j; // this lane's 64 bytes of BF16
    const int64_t warp = (int64_t(blockIdx.x) * THREADS + threadIdx.x) >> 5;
    const int64_t nwarps = (int64_t(gridDim.x) * THREADS) >> 5;
    int ti = warp < P.total_units ? locate_tensor(P, warp) : 0;
    // QF_Q4K_PREFETCH (BF16 input): the next unit's loads are issued before this unit is
    // encoded, so each warp keeps two units' loads in flight
    constexpr bool kPf = QF_Q4K_PREFETCH && kBf16;
    uint4 vn[4];
    auto load_raw = [&](int64_t u, int t, uint4 (&v)[4]) {
        const DevTensor& T = P.t[t];
        const int64_t e0 = (u - T.unit_begin) * 1024;
        const int64_t left = (T.numel - e0) >> 8;
        const int nsb = left < 4 ? (int)left : 4;
        const XT* xp = static_cast<const XT*>(T.x);
#pragma unroll
        for (int k = 0; k < 4; ++k)
            v[k] = k < nsb ? ld_stream<QF_Q4K_LD>(xp + e0 + 256 * k + 8 * lane) : make_uint4(0, 0, 0, 0);
    };
    if (kPf && warp < P.total_units) load_raw(warp, ti, vn);
    for (int64_t u = warp; u < P.total_units; u += nwarps) {
        ti = find_tensor(P, ti, u);
        const DevTensor& T = P.t[ti];
        const XT* xp = static_cast<const XT*>(T.x);
        const int64_t e0 = (u - T.unit_begin) * 1024;
        const int64_t left = (T.numel - e0) >> 8;
        const int nsb = left < 4 ? (int)left : 4;          // super-blocks in this unit
        const bool have = b < nsb;
        Elems<XT, 32> x;
        if constexpr (kBf16) {
            uint4 v[4];
            if constexpr (kPf) {
#pragma unroll
                for (int k = 0; k < 4; ++k) v[k] = vn[k];
                const int64_t un = u + nwarps;
                if (un < P.total_units) load_raw(un, find_tensor(P, ti, un), vn);
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    v[k] = k < nsb ? ld_stream<QF_Q4K_LD>(xp + e0 + 256 * k + 8 * lane) : make_uint4(0, 0, 0, 0);
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 4; ++k) sts128(sm_lane + k * kQ4kRow, v[k]);
            __syncwarp();
#pragma unroll
            for (int p = 0; p < 4; ++p) x.v[p] = lds128(sm_mine + 16 * p);
        } else {
            x.template load<1>(xp + e0 + 256 * b + 32 * j, have);
            __syncwarp();                                  // the previous unit's staging reads
        }
        const Q4kFit f = q4k_fit<XT, MSE>(x);
        if (MODE == 0) {
            q4k_emit_unit<XT>(T, e0, nsb, lane, x, f, sm_lane, sm_mine);
        } else {
            // clipped STE: keep grad where 0 <= (x + mm) * inv <= 15
            uint32_t keep = 0;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float t = __fmul_rn(__fadd_rn(x.get(k), f.mm), f.inv);
                keep |= (uint32_t)(t >= 0.0f && t <= 15.0f) << k;
            }
            uint4 v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                v[k] = k < nsb ? ld_stream<3>(T.g + e0 + 256 * k + 8 * lane) : make_uint4(0, 0, 0, 0);
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 4; ++k) sts128(sm_lane + k * kQ4kRow, v[k]);
            __syncwarp();
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                uint4 g = lds128(sm_mine + 16 * p);
                uint32_t gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int k = 8 * p + 2 * q;                 // elements k, k+1 of this lane
                    gw[q] = (((keep >> k) & 1u) ? (gw[q] & 0xFFFFu) : 0u) |
                            (((keep >> (k + 1)) & 1u) ? (gw[q] & 0xFFFF0000u) : 0u);
                }
                sts128(sm_mine + 16 * p, make_uint4(gw[0], gw[1], gw[2], gw[3]));
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < nsb) st_v4(T.y + e0 + 256 * k + 8 * lane, lds128(sm_lane + k * kQ4kRow));
        }
    }
}

// ------------------------------------------------------------------ tied amax
// Each CTA reduces one contiguous range of units, so a warp stays inside one tensor
// (one tie group) for many units; it keeps a running max |x| as FP32 bits and, on a
// group change and at the end, reduces across the warp and does one atomicMax on the
// group's FP32 bits (non-negative floats order like their bit patterns).
template <typename XT, int U, int MAXT, int THREADS>
__global__ void __launch_bounds__(THREADS) k_amax(const __grid_constant__ Table<MAXT> P) {
    // a programmatic dependent (the fused NVFP4 pass) may launch once every CTA of
    // this grid has started; it waits for this grid's results before reading them
    asm volatile("griddepcontrol.launch_dependents;");
    const int lane = threadIdx.x & 31;
    constexpr int kUnit = 256 * U;
    constexpr int kWarps = THREADS / 32;
#if QF_AMAX_ORDER == 0
    const int64_t per_cta = (P.total_units + gridDim.x - 1) / gridDim.x;
    const int64_t u_begin = int64_t(blockIdx.x) * per_cta;
    const int64_t u_end = min(u_begin + per_cta, P.total_units);
    const int64_t u_first = u_begin + (threadIdx.x >> 5);
    constexpr int64_t u_step = kWarps;
#else
    const int64_t u_end = P.total_units;
    const int64_t u_first = int64_t(blockIdx.x) * kWarps + (threadIdx.x >> 5);
    const int64_t u_step = int64_t(gridDim.x) * kWarps;
#endif
    float* amax = const_cast<float*>(P.group_amax);
    int ti = u_first < u_end ? locate_tensor(P, u_first) : 0;
    int g = -1;
    uint32_t run = 0;
    auto warp_max = [&]() {
        uint32_t a = run;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(kFull, a, o));
        return a;
    };
    auto publish = [&](int grp, uint32_t a) {
        atomicMax(reinterpret_cast<unsigned int*>(amax) + grp, a);
        if (P.tracked) atomicMax(reinterpret_cast<unsigned int*>(P.tracked) + grp, a);
    };
    // a warp that moves on to another tie group publishes the finished one at once
    auto flush = [&](int grp) {
        const uint32_t a = warp_max();
        if (lane == 0 && grp >= 0) publish(grp, a);
        run = 0;
    };
    for (int64_t u = u_first; u < u_end; u += u_step) {
        ti = find_tensor(P, ti, u);
        const DevTensor& T = P.t[ti];
        if (T.group != g) {
            if (g >= 0) flush(g);
            g = T.group;
        }
        const XT* x = static_cast<const XT*>(T.x);
        const int64_t e0 = (u - T.unit_begin) * kUnit;
        Elems<XT, 8> v[U];
#pragma unroll
        for (int s = 0; s < U; ++s) {
            const int64_t e = e0 + s * 256 + lane * 8;
            v[s].template load<QF_AMAX_LD>(x + e, e + 8 <= T.numel);
        }
#pragma unroll
        for (int s = 0; s < U; ++s) run = max(run, v[s].amax_bits());
    }
    // The warps' last groups are combined in the CTA first: when every CTA ends at
    // about the same time, thousands of same-address atomics would otherwise queue
    // at the end of the kernel (one per CTA and group remains).
    __shared__ int wgrp[kWarps];
    __shared__ uint32_t wmax[kWarps];
    const uint32_t a = warp_max();
    if (lane == 0) {
        wgrp[threadIdx.x >> 5] = g;
        wmax[threadIdx.x >> 5] = a;
    }
    __syncthreads();
    if (threadIdx.x < kWarps) {
        const int w = threadIdx.x, gw = wgrp[w];
        bool first = gw >= 0;                       // first warp of the CTA with this group
        uint32_t m = wmax[w];
        for (int o = 0; o < kWarps; ++o) {
            if (wgrp[o] != gw) continue;
            if (o < w) first = false;
            m = max(m, wmax[o]);
        }
        if (first) publish(gw, m);
    }
}

// amax of tensors whose element count is not a multiple of 8 handles the
// scalar tail here (one thread per leftover element; at most 7 per tensor).
template <typename XT, int MAXT>
__global__ void k_amax_tail(const __grid_constant__ Table<MAXT> P) {
    const int ti = blockIdx.x;
    if (ti >= P.n) return;
    const DevTensor& T = P.t[ti];
    const int64_t start = T.numel & ~int64_t(7);
    const int64_t e = start + threadIdx.x;
    if (threadIdx.x < 8 && e < T.numel) {
        uint32_t a;
        if constexpr (sizeof(XT) == 2)
            a = (uint32_t)(static_cast<const uint16_t*>(T.x)[e] & 0x7FFFu) << 16;
        else
            a = __float_as_uint(static_cast<const float*>(T.x)[e]) & 0x7FFFFFFFu;
        atomicMax(reinterpret_cast<unsigned int*>(const_cast<float*>(P.group_amax)) + T.group, a);
        if (P.tracked) atomicMax(reinterpret_cast<unsigned int*>(P.tracked) + T.group, a);
    }
}

// ------------------------------------------------------------------ STE identity
__global__ void __launch_bounds__(kThreads) k_copy(const uint16_t* __restrict__ src,
                                                   uint16_t* __restrict__ dst, int64_t n) {
    // one CTA per 4 * kThreads 16-byte vectors, all four loads in flight before the stores
    const int64_t nvec = n >> 3;
    const int64_t base = int64_t(blockIdx.x) * (4 * kThreads) + threadIdx.x;
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int64_t i = base + j * kThreads;
        if (i < nvec) v[j] = ld_stream<QF_COPY_LD>(src + 8 * i);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int64_t i = base + j * kThreads;
        if (i < nvec) st_v4(dst + 8 * i, v[j]);
    }
    if (blockIdx.x == 0 && threadIdx.x < (n & 7)) {
        const int64_t e = (nvec << 3) + threadIdx.x;
        dst[e] = src[e];
    }
}

}  // namespace qf
