// qf_lora.cuh -- LoRA-merged fake-quant on sm_100a (QATFactory project page, Method,
// "QAD": LoRA-QAD trains low-rank adapters on a frozen BF16 base and quantizes
// the merged weight W + scale * B A rather than W).
//
// The merged weight is formed on the fly and never written unless asked for:
//   acc = sum over k = 0..r-1, in increasing k, of B[i,k] * A[k,j]   (FP32)
//   M   = BF16(W[i,j] + scale * acc)
// A BF16 x BF16 product has at most 16 significant bits, so it is exact in FP32
// and one FMA per term rounds exactly like the separate multiply and add; the
// fixed order makes the result reproducible bit for bit (tensor cores are not
// used because their accumulation order is not specified).
//
// Layout: lane l owns 4 consecutive columns, a warp a 128-column slab, a CTA
// kLoraThreads / 32 slabs (1024 columns at 256 threads) by kLoraRows rows.  The warp keeps its A slab (r x 4 FP32)
// in registers across the CTA's rows; the CTA stages its kLoraRows rows of B in
// shared memory as FP32, so every B read is a broadcast.  W, y and codes accesses
// are contiguous 256-, 256- and 64-byte warp runs per row.
//
// The products run on sm_100's paired FP32 pipe: one fma.rn.f32x2 updates the
// accumulators of two adjacent columns, each rounded exactly as a scalar
// fma.rn.f32 would be (and, the products being exact, as a separate multiply and
// add would be).  B is stored in shared memory with every value twice, so one
// 16-byte load yields the (b, b) operand pairs of two consecutive k.
#pragma once

#include "qf_device.cuh"

namespace qf {

#ifndef QF_LORA_ROWS
#define QF_LORA_ROWS 64
#endif
constexpr int kLoraRows = QF_LORA_ROWS;   // rows per CTA unit (a multiple of 4)
#ifndef QF_LORA_THREADS
#define QF_LORA_THREADS 256
#endif
constexpr int kLoraThreads = QF_LORA_THREADS;
constexpr int kLoraCols = kLoraThreads / 32 * 128;   // columns per CTA unit (128 per warp)

// kLoraMergeAmax writes the merged weight like kLoraMerge and folds its max |M| into
// the tie-group amax like kLoraAmax, in one pass.
enum LoraMode { kLoraNV = 0, kLoraMX = 1, kLoraMerge = 2, kLoraAmax = 3, kLoraMergeAmax = 4 };

struct LoraTensor {
    const uint16_t* w;      // BF16 base [rows, cols]
    const uint16_t* b;      // BF16 [rows, rank]
    const uint16_t* a;      // BF16 [rank, cols]
    uint16_t* y;            // BF16 dequant (NV/MX) or merged weight (merge mode); nullable
    uint8_t* codes;         // packed E2M1 nibbles (nullable)
    uint8_t* scales;        // E4M3 / E8M0 bytes (nullable)
    int64_t rows, cols;
    int64_t unit_begin;     // first CTA unit of this tensor
    int64_t col_groups;     // ceil(cols / kLoraCols)
    int32_t rank;
    float scale;
    int32_t group;          // NVFP4 tie group
    int32_t pad;
};

template <int MAXT>
struct LoraTable {
    LoraTensor t[MAXT];
    int64_t total_units;
    const float* group_amax;    // NVFP4: tie-group amax (read); amax mode: output
    float* group_scale_out;     // NVFP4 s_t per group (nullable)
    int32_t n;
    int32_t n_groups;
};

template <int MAXT>
__device__ __forceinline__ int lora_locate(const LoraTable<MAXT>& P, int64_t u) {
    int lo = 0, hi = P.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.t[mid].unit_begin <= u) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// R: compile-time rank capacity (the runtime rank is <= R; A and B are zero-padded,
// which adds exact zeros to an accumulator that is never -0, so results do not change).
template <int MODE, int R, int MAXT>
__global__ void __launch_bounds__(kLoraThreads) k_lora(const __grid_constant__ LoraTable<MAXT> P) {
    __shared__ __align__(16) float2 bsm[kLoraRows][R];      // (b, b) pairs
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t cu = blockIdx.x;
    constexpr bool kWritesMerged = MODE == kLoraMerge || MODE == kLoraMergeAmax;
    constexpr bool kFoldsAmax = MODE == kLoraAmax || MODE == kLoraMergeAmax;
    if (MODE == kLoraNV && cu == 0 && P.group_scale_out) {
        for (int g = threadIdx.x; g < P.n_groups; g += kLoraThreads)
            P.group_scale_out[g] = nv_tensor_scale(P.group_amax[g]);
    }
    if (cu >= P.total_units) return;
    const LoraTensor& T = P.t[lora_locate(P, cu)];
    const int64_t local = cu - T.unit_begin;
    const int64_t r0 = (local / T.col_groups) * kLoraRows;
    const int64_t c_base = (local % T.col_groups) * kLoraCols;
    const int64_t rows_left = T.rows - r0;
    const int nrows = rows_left < kLoraRows ? (int)rows_left : kLoraRows;
    const int64_t col0 = c_base + wid * 128 + lane * 4;
    const bool colok = col0 < T.cols;          // cols % 16 == 0: a lane is all in or all out
    const int rank = T.rank;

    // this CTA's rows of B as FP32, zero-padded to R
    for (int idx = threadIdx.x; idx < kLoraRows * R; idx += kLoraThreads) {
        const int i = idx / R, k = idx % R;
        const float b = (i < nrows && k < rank) ? bf16_lo(T.b[(r0 + i) * rank + k]) : 0.0f;
        bsm[i][k] = make_float2(b, b);
    }
    // this lane's 4 columns of A as FP32 pairs (columns 0,1 and 2,3), zero-padded to R
    float2 a[R][2];
#pragma unroll
    for (int k = 0; k < R; ++k) {
        uint2 v = make_uint2(0, 0);
        if (k < rank && colok) v = *reinterpret_cast<const uint2*>(T.a + k * T.cols + col0);
        a[k][0] = make_float2(bf16_lo(v.x), bf16_hi(v.x));
        a[k][1] = make_float2(bf16_lo(v.y), bf16_hi(v.y));
    }
    __syncthreads();

    float s_t = 0.0f, six_st = 0.0f;
    if (MODE == kLoraNV) {
        s_t = nv_tensor_scale(P.group_amax[T.group]);
        six_st = __fmul_rn(6.0f, s_t);
    }
    uint32_t run = 0;                          // amax mode: running max |M| (FP32 bits)

    auto load_w = [&](int i0, uint2 (&wv)[4]) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const bool ok = colok && i0 + h < nrows;
            wv[h] = ok ? *reinterpret_cast<const uint2*>(T.w + (r0 + i0 + h) * T.cols + col0)
                       : make_uint2(0, 0);
        }
    };
    uint2 wcur[4], wnxt[4];
    load_w(0, wcur);
    for (int i0 = 0; i0 < nrows; i0 += 4) {
        if (i0 + 4 < nrows) load_w(i0 + 4, wnxt);          // the next 4 rows, in flight meanwhile
        // merged values of 4 rows x this lane's 4 columns
        float x[4][4];
        uint32_t xw[4][2];                                   // the same, as packed BF16 pairs
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const int i = min(i0 + h, nrows - 1);            // rows past the end are not stored
            float2 acc01 = make_float2(0.0f, 0.0f), acc23 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int k = 0; k < R; k += 2) {
                const float4 bk = *reinterpret_cast<const float4*>(&bsm[i][k]);
                const float2 b0 = make_float2(bk.x, bk.y), b1 = make_float2(bk.z, bk.w);
                acc01 = fma2_rn(b0, a[k][0], acc01);
                acc23 = fma2_rn(b0, a[k][1], acc23);
                acc01 = fma2_rn(b1, a[k + 1][0], acc01);
                acc23 = fma2_rn(b1, a[k + 1][1], acc23);
            }
            // scalar: a paired product must not feed an add (see mul2_rn)
            xw[h][0] = cvt_bf16x2(__fadd_rn(bf16_hi(wcur[h].x), __fmul_rn(T.scale, acc01.y)),
                                  __fadd_rn(bf16_lo(wcur[h].x), __fmul_rn(T.scale, acc01.x)));
            xw[h][1] = cvt_bf16x2(__fadd_rn(bf16_hi(wcur[h].y), __fmul_rn(T.scale, acc23.y)),
                                  __fadd_rn(bf16_lo(wcur[h].y), __fmul_rn(T.scale, acc23.x)));
            x[h][0] = bf16_lo(xw[h][0]); x[h][1] = bf16_hi(xw[h][0]);
            x[h][2] = bf16_lo(xw[h][1]); x[h][3] = bf16_hi(xw[h][1]);
        }
        if (kWritesMerged) {
#pragma unroll
            for (int h = 0; h < 4; ++h)
                if (colok && i0 + h < nrows && T.y)
                    *reinterpret_cast<uint2*>(T.y + (r0 + i0 + h) * T.cols + col0) =
                        make_uint2(xw[h][0], xw[h][1]);
        }
        if (MODE != kLoraMerge) {
            uint32_t m[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                m[h] = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) m[h] = max(m[h], __float_as_uint(x[h][c]) & 0x7FFFFFFFu);
            }
            if (kFoldsAmax) {
#pragma unroll
                for (int h = 0; h < 4; ++h)
                    if (i0 + h < nrows) run = max(run, m[h]);
            } else {
                // block max over the 4 (NVFP4, 16 elements) or 8 (MXFP4, 32) lanes of the block
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    m[h] = max(m[h], __shfl_xor_sync(kFull, m[h], 1));
                    m[h] = max(m[h], __shfl_xor_sync(kFull, m[h], 2));
                    if (MODE == kLoraMX) m[h] = max(m[h], __shfl_xor_sync(kFull, m[h], 4));
                }
                float S[4], inv[4];
                uint32_t sbyte[4];
                if (MODE == kLoraNV) {
                    // the 4 lanes of a block each derive one of the 4 rows' scales, then share
                    const int t = lane & 3;
                    const uint32_t mt = t == 0 ? m[0] : t == 1 ? m[1] : t == 2 ? m[2] : m[3];
                    uint32_t sb_t;
                    float S_t, inv_t;
                    nv_block_scale(__uint_as_float(mt), s_t, six_st, sb_t, S_t, inv_t);
                    const int base = lane & ~3;
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        sbyte[h] = __shfl_sync(kFull, sb_t, base + h);
                        S[h] = __shfl_sync(kFull, S_t, base + h);
                        inv[h] = __shfl_sync(kFull, inv_t, base + h);
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const uint32_t E = m[h] >> 23;
                        sbyte[h] = E > 2u ? E - 2u : 0u;
                        inv[h] = __uint_as_float((254u - sbyte[h]) << 23);
                        S[h] = sbyte[h] ? __uint_as_float(sbyte[h] << 23) : __uint_as_float(0x00200000u);
                    }
                }
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 inv2 = make_float2(inv[h], inv[h]);
                    const float2 q01 = mul2_rn(make_float2(x[h][0], x[h][1]), inv2);
                    const float2 q23 = mul2_rn(make_float2(x[h][2], x[h][3]), inv2);
                    float q[4] = {q01.x, q01.y, q23.x, q23.y};
                    if (MODE == kLoraNV && __builtin_expect(isinf(inv[h]), 0)) {
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            if (x[h][c] == 0.0f) q[c] = x[h][c];
                    }
                    const uint32_t b0 = cvt_e2m1x2(q[1], q[0]), b1 = cvt_e2m1x2(q[3], q[2]);
                    if (!colok || i0 + h >= nrows) continue;
                    const int64_t e = (r0 + i0 + h) * T.cols + col0;   // flat element index
                    if (T.y) {
                        const uint32_t h0 = cvt_e2m1x2_f16x2(b0), h1 = cvt_e2m1x2_f16x2(b1);
                        const float2 S2 = make_float2(S[h], S[h]);
                        const float2 d01 = mul2_rn(make_float2(f16_lo(h0), f16_hi(h0)), S2);
                        const float2 d23 = mul2_rn(make_float2(f16_lo(h1), f16_hi(h1)), S2);
                        *reinterpret_cast<uint2*>(T.y + e) =
                            make_uint2(cvt_bf16x2(d01.y, d01.x), cvt_bf16x2(d23.y, d23.x));
                    }
                    if (T.codes)
                        *reinterpret_cast<uint16_t*>(T.codes + (e >> 1)) = (uint16_t)(b0 | (b1 << 8));
                    if (T.scales && (lane & (MODE == kLoraNV ? 3 : 7)) == 0)
                        T.scales[e >> (MODE == kLoraNV ? 4 : 5)] = (uint8_t)sbyte[h];
                }
            }
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) wcur[h] = wnxt[h];
    }
    if (kFoldsAmax) {
        // one atomic per CTA (its unit lies in one tensor), not one per warp
        __shared__ uint32_t wmax[kLoraThreads / 32];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) run = max(run, __shfl_xor_sync(kFull, run, o));
        if (lane == 0) wmax[wid] = run;
        __syncthreads();
        if (threadIdx.x == 0) {
            for (int w = 1; w < kLoraThreads / 32; ++w) run = max(run, wmax[w]);
            if (run != 0)
                atomicMax(reinterpret_cast<unsigned int*>(const_cast<float*>(P.group_amax)) + T.group,
                          run);
        }
    }
}

}  // namespace qf
