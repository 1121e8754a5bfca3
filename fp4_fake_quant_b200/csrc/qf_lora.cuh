// qf_lora.cuh -- LoRA-merged fake-quant on sm_100a (QATFactory project page, Method,
// "QAD": LoRA-QAD trains low-rank adapters on a frozen BF16 base and quantizes
// the merged weight W + scale * B A rather than W).
//
// The merged weight is formed on the fly and never written unless asked for:
//   acc = sum over k = 0..r-1, in increasing k, of B[i,k] * A[k,j]   (FP32)
//   M   = BF16(W[i,j] + scale * acc)
// Each term is one fused multiply-add (acc + b*a rounded once; a BF16 x BF16 product
// has at most 16 significant bits, so this is also the separate multiply and add
// unless the product underflows); the fixed order makes the result reproducible bit
// for bit (tensor cores are not used because their accumulation order is not
// specified).
//
// Layout: lane l owns 4 consecutive columns, a warp a 128-column slab, a CTA
// kLoraThreads / 32 slabs (1024 columns at 256 threads) by kLoraRows rows.  The warp
// keeps its A slab (r x 4 FP32) in registers across the CTA's rows; the CTA stages its
// kLoraRows rows of B in shared memory as FP32, so every B read is a broadcast.  W, y
// and codes accesses are contiguous 256-, 256- and 64-byte warp runs per row.
//
// The products run on sm_100's paired FP32 pipe: one fma.rn.f32x2 updates the
// accumulators of two adjacent columns, each rounded exactly as a scalar
// fma.rn.f32 would be.  Operands and accumulators live in 64-bit registers from load to
// use, so no pair is ever repacked.  B is stored in shared memory with every value
// twice, so one 16-byte load yields the (b, b) operand pairs of two consecutive k.
//
// W arrives 4 rows per step.  The merge and amax modes, whose arithmetic per byte is
// lightest, keep QF_LORA_STAGES steps of it in flight through a per-lane cp.async
// ring in shared memory (each lane reads back only what it copied, so the ring needs
// no barrier and its waits are the hardware's cp.async.wait_group); the quantizing
// modes load the next step into registers and prefetch further rows to L2.  Whole
// tiles of the merge and amax modes run a guard-free copy of the row loop.  Maxima
// are taken on the packed BF16 merged values, two 16-bit magnitudes at a time.
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
#ifndef QF_LORA_STAGES
#define QF_LORA_STAGES 4        // merge / amax modes: W ring depth in 4-row steps (cp.async)
#endif
#ifndef QF_LORA_NV_STAGES
#define QF_LORA_NV_STAGES 0     // NVFP4 / MXFP4 modes: the same (0: register prefetch)
#endif
#ifndef QF_LORA_PF
#define QF_LORA_PF 4            // with register prefetch: L2 prefetch distance, 4-row steps
#endif
#ifndef QF_LORA_PIPE
#define QF_LORA_PIPE 1          // merge modes: the software-pipelined 2-row loop (unit_pipe)
#endif
#ifndef QF_LORA_FUSED
#define QF_LORA_FUSED 1         // pipelined merge: one fused rounding where scale = 2^e, e >= 0
#endif
#ifndef QF_LORA_FULL
#define QF_LORA_FULL 1          // guard-free copy of the unit loop for whole tiles: 0 none,
#endif                          // 1 merge / amax modes, 2 every mode

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

// Packed FP32 pairs kept in 64-bit registers from load to use, so the paired pipe's
// operands need no repacking: lo = the pair's first (lower-address) value.
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
__device__ __forceinline__ float2 unpk2(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
// d = a * b + c on both halves, each rounded once (fused: the product is not rounded)
__device__ __forceinline__ uint64_t fma2_pk(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// per-half unsigned 16-bit max: the max |v| of BF16 pairs once their sign bits are cleared
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
// FP32 bits of the larger of the two BF16 magnitudes in a max_u16x2 result
__device__ __forceinline__ uint32_t bf16x2_max_bits(uint32_t m) {
    return max(m & 0xFFFFu, m >> 16) << 16;
}


template <bool B>
struct FullTile { static constexpr bool value = B; };

// R: compile-time rank capacity (the runtime rank is <= R; A and B are zero-padded,
// which adds exact zeros to an accumulator that is never -0, so results do not change).
template <int MODE, int R, int MAXT>
__global__ void __launch_bounds__(kLoraThreads, R <= 16 ? 2 : 1) k_lora(const __grid_constant__ LoraTable<MAXT> P) {
    __shared__ __align__(16) uint64_t bsm[kLoraRows][R];     // (b, b) FP32 pairs
    // W ring: every lane copies its own 8 bytes of each row into its own slots and reads
    // only those back, so the ring needs no barrier (48 KB of static shared memory caps
    // the depth at rank 32)
    constexpr int kWantStages = MODE == kLoraNV || MODE == kLoraMX ? QF_LORA_NV_STAGES
                                                                   : QF_LORA_STAGES;
    constexpr int kStages = R > 16 && kWantStages > 3 ? 3 : kWantStages;
    constexpr int kPf = kStages == 0 ? QF_LORA_PF : 0;
    constexpr int kRing = kStages > 0 ? kStages : 1;
    __shared__ __align__(16) uint2 wring[kRing][4][kLoraThreads];
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
    const int64_t cols = T.cols;
    const int64_t col0 = c_base + wid * 128 + lane * 4;
    const bool colok = col0 < cols;            // cols % 16 == 0: a lane is all in or all out
    const int rank = T.rank;
    const float scale = T.scale;

    // with register prefetch, W rows reach L2 kPf 4-row steps before the step that
    // loads them: the warp's slab of a row is 256 bytes (fewer at the last column
    // group), two lines, one lane each
    const int64_t wcol0 = c_base + wid * 128;
    const int pf_bytes = wcol0 < cols ? (int)(min(cols - wcol0, (int64_t)128) * 2) : 0;
    const uint16_t* wslab = T.w + r0 * cols + wcol0;
    if (kPf > 0) {
        for (int rr = lane >> 1; rr < 4 * kPf; rr += 16)
            if (128 * (lane & 1) < pf_bytes && 4 + rr < nrows)
                prefetch_line_l2(wslab + (4 + rr) * cols + 64 * (lane & 1));
    }

    // this CTA's rows of B as FP32, zero-padded to R
    for (int idx = threadIdx.x; idx < kLoraRows * R; idx += kLoraThreads) {
        const int i = idx / R, k = idx % R;
        const float b = (i < nrows && k < rank) ? bf16_lo(T.b[(r0 + i) * rank + k]) : 0.0f;
        bsm[i][k] = pk2(b, b);
    }
    // this lane's 4 columns of A as FP32 pairs (columns 0,1 and 2,3), zero-padded to R
    uint64_t a[R][2];
#pragma unroll
    for (int k = 0; k < R; ++k) {
        uint2 v = make_uint2(0, 0);
        if (k < rank && colok) v = *reinterpret_cast<const uint2*>(T.a + k * cols + col0);
        a[k][0] = pk2(bf16_lo(v.x), bf16_hi(v.x));
        a[k][1] = pk2(bf16_lo(v.y), bf16_hi(v.y));
    }
    __syncthreads();

    float s_t = 0.0f, six_st = 0.0f;
    if (MODE == kLoraNV) {
        s_t = nv_tensor_scale(P.group_amax[T.group]);
        six_st = __fmul_rn(6.0f, s_t);
    }
    uint32_t run = 0;                          // amax modes: max |M| so far, per BF16 half

    // One CTA unit: FULL when all kLoraRows rows exist and the lane's columns do, so no
    // access needs a guard.  Otherwise rows past the end re-read the last row (their
    // merged values repeat that row's, which leaves every max unchanged, and they are
    // never stored) and a lane past the last column reads zeros (merged value +0).
    const uint16_t* wbase = T.w + r0 * cols + col0;
    auto unit = [&](auto tag) {
        constexpr bool FULL = decltype(tag)::value;
        const int n = FULL ? kLoraRows : nrows;
        auto row = [&](int i) { return FULL ? i : min(i, n - 1); };
        auto load_w = [&](int i0, uint2 (&wv)[4]) {
#pragma unroll
            for (int h = 0; h < 4; ++h)
                wv[h] = (FULL || colok)
                            ? *reinterpret_cast<const uint2*>(wbase + row(i0 + h) * cols)
                            : make_uint2(0, 0);
        };
        const uint32_t ring = (uint32_t)__cvta_generic_to_shared(&wring[0][0][threadIdx.x]);
        // rows 4 it .. 4 it + 3 into ring stage it % kStages (one copy group per step,
        // empty past the last row, so the group count stays uniform)
        auto issue = [&](int it) {
            if (4 * it < n) {
                const uint32_t dst = ring + (uint32_t)((it % kRing) * 4 * kLoraThreads * 8);
#pragma unroll
                for (int h = 0; h < 4; ++h)
                    cp_async8(dst + h * kLoraThreads * 8,
                              (FULL || colok) ? (const void*)(wbase + row(4 * it + h) * cols)
                                              : (const void*)T.w,
                              (FULL || colok) ? 8u : 0u);
            }
            cp_async_commit();
        };
        uint2 wcur[4], wnxt[4];
        if constexpr (kStages > 0) {
#pragma unroll
            for (int st = 0; st < kStages - 1; ++st) issue(st);
        } else {
            load_w(0, wcur);
        }
#pragma unroll 1
        for (int i0 = 0; i0 < n; i0 += 4) {
            if constexpr (kStages > 0) {
                const int it = i0 >> 2;
                cp_async_wait<kStages - 2>();              // this step's group has landed
                const uint32_t src = ring + (uint32_t)((it % kRing) * 4 * kLoraThreads * 8);
#pragma unroll
                for (int h = 0; h < 4; ++h) wcur[h] = lds64(src + h * kLoraThreads * 8);
                issue(it + kStages - 1);                   // refills the stage read last step
            }
            if (kPf > 0 && lane < 8) {
                const int rr = i0 + 4 + 4 * kPf + (lane >> 1);
                if (128 * (lane & 1) < pf_bytes && rr < nrows)
                    prefetch_line_l2(wslab + rr * cols + 64 * (lane & 1));
            }
            if (kStages == 0 && i0 + 4 < n) load_w(i0 + 4, wnxt);   // next 4 rows, in flight
            // merged values of 4 rows x this lane's 4 columns, as packed BF16 pairs
            uint32_t xw[4][2];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const int i = row(i0 + h);
                uint64_t acc01 = 0, acc23 = 0;           // (+0, +0)
#pragma unroll
                for (int k = 0; k < R; k += 2) {
                    const ulonglong2 bk = *reinterpret_cast<const ulonglong2*>(&bsm[i][k]);
                    acc01 = fma2_pk(bk.x, a[k][0], acc01);
                    acc23 = fma2_pk(bk.x, a[k][1], acc23);
                    acc01 = fma2_pk(bk.y, a[k + 1][0], acc01);
                    acc23 = fma2_pk(bk.y, a[k + 1][1], acc23);
                }
                // scalar: a paired product must not feed an add (see mul2_rn)
                const float2 s01 = unpk2(acc01), s23 = unpk2(acc23);
                xw[h][0] = cvt_bf16x2(__fadd_rn(bf16_hi(wcur[h].x), __fmul_rn(scale, s01.y)),
                                      __fadd_rn(bf16_lo(wcur[h].x), __fmul_rn(scale, s01.x)));
                xw[h][1] = cvt_bf16x2(__fadd_rn(bf16_hi(wcur[h].y), __fmul_rn(scale, s23.y)),
                                      __fadd_rn(bf16_lo(wcur[h].y), __fmul_rn(scale, s23.x)));
            }
            if (kWritesMerged) {
#pragma unroll
                for (int h = 0; h < 4; ++h)
                    if (FULL || (colok && i0 + h < n))
                        *reinterpret_cast<uint2*>(T.y + (r0 + i0 + h) * cols + col0) =
                            make_uint2(xw[h][0], xw[h][1]);
            }
            if (kFoldsAmax) {
#pragma unroll
                for (int h = 0; h < 4; ++h)
                    run = max_u16x2(run, max_u16x2(xw[h][0] & 0x7FFF7FFFu, xw[h][1] & 0x7FFF7FFFu));
            } else if (MODE == kLoraNV || MODE == kLoraMX) {
                // block max over the 4 (NVFP4, 16 elements) or 8 (MXFP4, 32) lanes of the block
                uint32_t m[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    m[h] = bf16x2_max_bits(max_u16x2(xw[h][0] & 0x7FFF7FFFu, xw[h][1] & 0x7FFF7FFFu));
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
                        S[h] = sbyte[h] ? __uint_as_float(sbyte[h] << 23) : __uint_as_float(0x00400000u);
                    }
                }
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float x[4] = {bf16_lo(xw[h][0]), bf16_hi(xw[h][0]),
                                        bf16_lo(xw[h][1]), bf16_hi(xw[h][1])};
                    const float2 inv2 = make_float2(inv[h], inv[h]);
                    const float2 q01 = mul2_rn(make_float2(x[0], x[1]), inv2);
                    const float2 q23 = mul2_rn(make_float2(x[2], x[3]), inv2);
                    float q[4] = {q01.x, q01.y, q23.x, q23.y};
                    if (MODE == kLoraNV && __builtin_expect(isinf(inv[h]), 0)) {
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            if (x[c] == 0.0f) q[c] = x[c];
                    }
                    const uint32_t b0 = cvt_e2m1x2(q[1], q[0]), b1 = cvt_e2m1x2(q[3], q[2]);
                    if (!FULL && (!colok || i0 + h >= n)) continue;
                    const int64_t e = (r0 + i0 + h) * cols + col0;   // flat element index
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
            if constexpr (kStages == 0) {
#pragma unroll
                for (int h = 0; h < 4; ++h) wcur[h] = wnxt[h];
            }
        }
        if constexpr (kStages > 0) cp_async_wait<0>();
    };
    // Merge modes, software-pipelined over 2-row steps: each iteration forms the rank-r
    // products of the next two rows while it finishes the current two (merge with W,
    // BF16 rounding, store, max), so within every warp the FMA pipe's work and the rest
    // interleave instead of alternating in bursts.  W comes through the same per-lane
    // cp.async ring, viewed as 2-row stages (twice as many).
    auto unit_pipe = [&](auto tag, auto ftag) {
        constexpr bool FULL = decltype(tag)::value;
        constexpr bool FUSED = decltype(ftag)::value;   // W + scale * acc in one rounding
        const uint64_t s2 = pk2(scale, scale);
        constexpr int kS = 2 * kRing;                   // ring depth in 2-row steps
        const int n = FULL ? kLoraRows : nrows;
        const int nst = (n + 1) >> 1;
        auto row = [&](int i) { return FULL ? i : min(i, n - 1); };
        const uint32_t ring = (uint32_t)__cvta_generic_to_shared(&wring[0][0][threadIdx.x]);
        auto issue = [&](int st) {
            if (st < nst) {
                const uint32_t dst = ring + (uint32_t)((st % kS) * 2 * kLoraThreads * 8);
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    cp_async8(dst + h * kLoraThreads * 8,
                              (FULL || colok) ? (const void*)(wbase + row(2 * st + h) * cols)
                                              : (const void*)T.w,
                              (FULL || colok) ? 8u : 0u);
            }
            cp_async_commit();
        };
        auto chains = [&](int st, uint64_t (&acc)[2][2]) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int i = row(2 * st + h);
                acc[h][0] = 0;
                acc[h][1] = 0;
#pragma unroll
                for (int k = 0; k < R; k += 2) {
                    const ulonglong2 bk = *reinterpret_cast<const ulonglong2*>(&bsm[i][k]);
                    acc[h][0] = fma2_pk(bk.x, a[k][0], acc[h][0]);
                    acc[h][1] = fma2_pk(bk.x, a[k][1], acc[h][1]);
                    acc[h][0] = fma2_pk(bk.y, a[k + 1][0], acc[h][0]);
                    acc[h][1] = fma2_pk(bk.y, a[k + 1][1], acc[h][1]);
                }
            }
        };
        uint16_t* yrow = kWritesMerged ? T.y + r0 * cols + col0 : nullptr;
        // one step: the next rows' products into nxt, this step's rows finished from cur
        auto step = [&](int st, uint64_t (&cur)[2][2], uint64_t (&nxt)[2][2]) {
            cp_async_wait<kS - 2>();                    // this step's W has landed
            const uint32_t src = ring + (uint32_t)((st % kS) * 2 * kLoraThreads * 8);
            const uint2 w[2] = {lds64(src), lds64(src + kLoraThreads * 8)};
            issue(st + kS - 1);                         // refills the stage read last step
            if (st + 1 < nst) chains(st + 1, nxt);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t x0, x1;
                if constexpr (FUSED) {
                    // scale * acc is exact here (see kFusedMerge), so one fused rounding of
                    // W + scale * acc equals the rounded product followed by the rounded add
                    const float2 m01 = unpk2(fma2_pk(s2, cur[h][0],
                                                     pk2(bf16_lo(w[h].x), bf16_hi(w[h].x))));
                    const float2 m23 = unpk2(fma2_pk(s2, cur[h][1],
                                                     pk2(bf16_lo(w[h].y), bf16_hi(w[h].y))));
                    x0 = cvt_bf16x2(m01.y, m01.x);
                    x1 = cvt_bf16x2(m23.y, m23.x);
                } else {
                    // scalar: a paired product must not feed an add (see mul2_rn)
                    const float2 s01 = unpk2(cur[h][0]), s23 = unpk2(cur[h][1]);
                    x0 = cvt_bf16x2(__fadd_rn(bf16_hi(w[h].x), __fmul_rn(scale, s01.y)),
                                    __fadd_rn(bf16_lo(w[h].x), __fmul_rn(scale, s01.x)));
                    x1 = cvt_bf16x2(__fadd_rn(bf16_hi(w[h].y), __fmul_rn(scale, s23.y)),
                                    __fadd_rn(bf16_lo(w[h].y), __fmul_rn(scale, s23.x)));
                }
                if (kWritesMerged && (FULL || (colok && 2 * st + h < n)))
                    *reinterpret_cast<uint2*>(yrow + h * cols) = make_uint2(x0, x1);
                if (kFoldsAmax)
                    run = max_u16x2(run, max_u16x2(x0 & 0x7FFF7FFFu, x1 & 0x7FFF7FFFu));
            }
            if (kWritesMerged) yrow += 2 * cols;
        };
#pragma unroll
        for (int st = 0; st < kS - 1; ++st) issue(st);
        uint64_t accA[2][2], accB[2][2];
        chains(0, accA);
#pragma unroll 1
        for (int st = 0; st < nst; st += 2) {           // two steps per pass: the
            step(st, accA, accB);                       // accumulators swap roles
            if (st + 1 < nst) step(st + 1, accB, accA);
        }
        cp_async_wait<0>();
    };
    constexpr bool kSplitFull = QF_LORA_FULL == 2 || (QF_LORA_FULL == 1 && MODE != kLoraNV &&
                                                      MODE != kLoraMX);
    constexpr bool kPipe = QF_LORA_PIPE && kStages > 0 && (MODE == kLoraMerge ||
                                                            MODE == kLoraMergeAmax);
    if constexpr (kPipe) {
        // kFusedMerge: with scale = 2^e, e >= 0, scale * acc is exact unless it overflows;
        // |acc| <= sum_k |b_k| |a_k| (1 + 2^-20) <= Rmax Cmax (1 + 2^-20) over the CTA's
        // rows and columns, so scale Rmax Cmax (1 + 2^-6) < 2^126 rules the overflow out
        // and the merge may round W + scale * acc once (a paired FMA per two elements)
        __shared__ uint32_t s_rmax, s_cmax;
        if (threadIdx.x == 0) s_rmax = s_cmax = 0u;
        __syncthreads();
        if (threadIdx.x < kLoraRows) {
            float r = 0.0f;
#pragma unroll
            for (int k = 0; k < R; ++k) r = __fadd_rn(r, fabsf(unpk2(bsm[threadIdx.x][k]).x));
            atomicMax(&s_rmax, __float_as_uint(r));
        }
        uint32_t cm = 0;
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const float2 p = unpk2(a[k][0]), q = unpk2(a[k][1]);
            cm = max(cm, max(max(__float_as_uint(p.x), __float_as_uint(p.y)),
                             max(__float_as_uint(q.x), __float_as_uint(q.y))) & 0x7FFFFFFFu);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cm = max(cm, __shfl_xor_sync(kFull, cm, o));
        if (lane == 0) atomicMax(&s_cmax, cm);
        __syncthreads();
        const uint32_t sb = __float_as_uint(scale);
        const bool pow2 = (sb & 0x807FFFFFu) == 0u && (sb >> 23) >= 127u && (sb >> 23) < 255u;
        const float bound = __fmul_rn(__fmul_rn(__fmul_rn(scale, __uint_as_float(s_rmax)),
                                                __uint_as_float(s_cmax)), 1.0f + 0x1p-6f);
        const bool fused = QF_LORA_FUSED && pow2 && bound < 0x1p126f;
        if (nrows == kLoraRows && colok) {
            if (fused) unit_pipe(FullTile<true>{}, FullTile<true>{});
            else unit_pipe(FullTile<true>{}, FullTile<false>{});
        } else {
            if (fused) unit_pipe(FullTile<false>{}, FullTile<true>{});
            else unit_pipe(FullTile<false>{}, FullTile<false>{});
        }
    } else {
        if (kSplitFull && nrows == kLoraRows && colok) unit(FullTile<true>{});
        else unit(FullTile<false>{});
    }

    if (kFoldsAmax) {
        // one atomic per CTA (its unit lies in one tensor), not one per warp
        __shared__ uint32_t wmax[kLoraThreads / 32];
        run = bf16x2_max_bits(run);
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


// ------------------------------------------------------------------ merge, 8 columns per lane
// k_lora8: the merge modes (kLoraMerge, kLoraMergeAmax) and the NVFP4 mode for rank
// <= 16 with each lane owning 8 consecutive columns (a 128-thread CTA still covers 1024
// columns by kLora8Rows rows).  Against 4 columns per lane, every broadcast
// load of two (b, b) pairs feeds 8 paired FMAs instead of 4 and the per-row work is
// shared by twice the elements; the A slab takes 128 registers per lane (R = 16).
// Arithmetic, results and the fused-rounding rule are those of k_lora's merge.  In the
// NVFP4 mode a 16-element block spans a lane pair, and the merged BF16 values of each
// row go through the 8-element-lane NVFP4 codec (fp4_lane): block max over the pair,
// E4M3 block scale, E2M1 codes and the dequantized BF16 values, as in k_lora.
#ifndef QF_LORA8
#define QF_LORA8 1
#endif
#ifndef QF_LORA8_NV
#define QF_LORA8_NV 1           // NVFP4 mode of the merge-on-the-fly pass in k_lora8
#endif
#ifndef QF_LORA8_NV_MINB
#define QF_LORA8_NV_MINB 2
#endif
#ifndef QF_LORA8_TAB
#define QF_LORA8_TAB 1          // NVFP4 mode: block scales from the CTA's tables (nv_block_scale_tab)
#endif
#ifndef QF_LORA8_STAGES
#define QF_LORA8_STAGES 4       // W ring depth in 2-row steps (16 bytes per lane and row)
#endif
#ifndef QF_LORA8_MINB
#define QF_LORA8_MINB 3
#endif
constexpr int kLora8Threads = 128;
#ifndef QF_LORA8_ROWS
#define QF_LORA8_ROWS 64
#endif
constexpr int kLora8Rows = QF_LORA8_ROWS;   // rows per CTA unit of k_lora8 (an even number)

__device__ __forceinline__ void cp_async16_cg(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes) : "memory");
}

template <int MODE, int R, int MAXT>
__global__ void __launch_bounds__(kLora8Threads, MODE == kLoraNV ? QF_LORA8_NV_MINB : QF_LORA8_MINB)
    k_lora8(const __grid_constant__ LoraTable<MAXT> P) {
    static_assert(MODE == kLoraMerge || MODE == kLoraMergeAmax || MODE == kLoraNV,
                  "merge modes and NVFP4 only");
    static_assert(R <= 16, "the A slab of rank 32 does not fit in registers");
    constexpr int kS = QF_LORA8_STAGES;
    constexpr bool kNV = MODE == kLoraNV;
    constexpr bool kWritesMerged = !kNV;
    constexpr bool kFoldsAmax = MODE == kLoraMergeAmax;
    __shared__ __align__(16) uint64_t bsm[kLora8Rows][R];                 // (b, b) FP32 pairs
    __shared__ __align__(16) uint4 wring[kS][2][kLora8Threads];
    __shared__ uint32_t s_rmax, s_cmax;
    __shared__ NvScaleTab s_tab[1];                                        // NVFP4 mode
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t cu = blockIdx.x;
    if (kNV && cu == 0 && P.group_scale_out) {
        for (int g = threadIdx.x; g < P.n_groups; g += kLora8Threads)
            P.group_scale_out[g] = nv_tensor_scale(P.group_amax[g]);
    }
    if (cu >= P.total_units) return;
    const LoraTensor& T = P.t[lora_locate(P, cu)];
    const int64_t local = cu - T.unit_begin;
    const int64_t r0 = (local / T.col_groups) * kLora8Rows;
    const int64_t c_base = (local % T.col_groups) * kLoraCols;
    const int64_t rows_left = T.rows - r0;
    const int nrows = rows_left < kLora8Rows ? (int)rows_left : kLora8Rows;
    const int64_t cols = T.cols;
    const int64_t col0 = c_base + wid * 256 + lane * 8;
    const bool colok = col0 < cols;            // cols % 16 == 0: 8 columns all in or all out
    const int rank = T.rank;
    const float scale = T.scale;

    for (int idx = threadIdx.x; idx < kLora8Rows * R; idx += kLora8Threads) {
        const int i = idx / R, k = idx % R;
        const float b = (i < nrows && k < rank) ? bf16_lo(T.b[(r0 + i) * rank + k]) : 0.0f;
        bsm[i][k] = pk2(b, b);
    }
    // this lane's 8 columns of A as four FP32 pairs per k, zero-padded to R
    uint64_t a[R][4];
#pragma unroll
    for (int k = 0; k < R; ++k) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (k < rank && colok) v = *reinterpret_cast<const uint4*>(T.a + k * cols + col0);
        a[k][0] = pk2(bf16_lo(v.x), bf16_hi(v.x));
        a[k][1] = pk2(bf16_lo(v.y), bf16_hi(v.y));
        a[k][2] = pk2(bf16_lo(v.z), bf16_hi(v.z));
        a[k][3] = pk2(bf16_lo(v.w), bf16_hi(v.w));
    }
    if (threadIdx.x == 0) s_rmax = s_cmax = 0u;
    float s_t = 0.0f, six_st = 0.0f, yd = 0.0f;
    if (kNV) {
        s_t = nv_tensor_scale(P.group_amax[T.group]);
        six_st = __fmul_rn(6.0f, s_t);
        if (QF_LORA8_TAB) {
            yd = nv_ratio_recip(six_st);
            if (yd != 0.0f) nv_tab_fill(s_tab[0], s_t, threadIdx.x, kLora8Threads);
        }
    }
    __syncthreads();
    // the fused-rounding rule of k_lora (kFusedMerge): scale = 2^e, e >= 0, and
    // scale * Rmax * Cmax * (1 + 2^-6) < 2^126 over the CTA's rows and columns
    if (threadIdx.x < kLora8Rows) {
        float r = 0.0f;
#pragma unroll
        for (int k = 0; k < R; ++k) r = __fadd_rn(r, fabsf(unpk2(bsm[threadIdx.x][k]).x));
        atomicMax(&s_rmax, __float_as_uint(r));
    }
    uint32_t cm = 0;
#pragma unroll
    for (int k = 0; k < R; ++k)
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 q = unpk2(a[k][p]);
            cm = max(cm, max(__float_as_uint(q.x), __float_as_uint(q.y)) & 0x7FFFFFFFu);
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cm = max(cm, __shfl_xor_sync(kFull, cm, o));
    if (lane == 0) atomicMax(&s_cmax, cm);
    __syncthreads();
    const uint32_t sbits = __float_as_uint(scale);
    const bool pow2 = (sbits & 0x807FFFFFu) == 0u && (sbits >> 23) >= 127u && (sbits >> 23) < 255u;
    const float bound = __fmul_rn(__fmul_rn(__fmul_rn(scale, __uint_as_float(s_rmax)),
                                            __uint_as_float(s_cmax)), 1.0f + 0x1p-6f);
    const bool fused = QF_LORA_FUSED && pow2 && bound < 0x1p126f;

    uint32_t run = 0;
    const uint16_t* wbase = T.w + r0 * cols + col0;
    auto unit = [&](auto tag, auto ftag) {
        constexpr bool FULL = decltype(tag)::value;
        constexpr bool FUSED = decltype(ftag)::value;
        const uint64_t s2 = pk2(scale, scale);
        const int n = FULL ? kLora8Rows : nrows;
        const int nst = (n + 1) >> 1;
        auto row = [&](int i) { return FULL ? i : min(i, n - 1); };
        const uint32_t ring = (uint32_t)__cvta_generic_to_shared(&wring[0][0][threadIdx.x]);
        auto issue = [&](int st) {
            if (st < nst) {
                const uint32_t dst = ring + (uint32_t)((st % kS) * 2 * kLora8Threads * 16);
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    cp_async16_cg(dst + h * kLora8Threads * 16,
                                  (FULL || colok) ? (const void*)(wbase + row(2 * st + h) * cols)
                                                  : (const void*)T.w,
                                  (FULL || colok) ? 16u : 0u);
            }
            cp_async_commit();
        };
#pragma unroll
        for (int st = 0; st < kS - 1; ++st) issue(st);
        // the merge modes step a row pointer; the NVFP4 mode a flat element index
        uint16_t* yrow = kWritesMerged ? T.y + r0 * cols + col0 : nullptr;
        int64_t erow = kNV ? r0 * cols + col0 : 0;
#pragma unroll 1
        for (int st = 0; st < nst; ++st) {
            cp_async_wait<kS - 2>();                        // this step's W has landed
            const uint32_t src = ring + (uint32_t)((st % kS) * 2 * kLora8Threads * 16);
            const uint4 w[2] = {lds128(src), lds128(src + kLora8Threads * 16)};
            issue(st + kS - 1);                             // refills the stage read last step
            uint64_t acc[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int i = row(2 * st + h);
#pragma unroll
                for (int p = 0; p < 4; ++p) acc[h][p] = 0;
#pragma unroll
                for (int k = 0; k < R; k += 2) {
                    const ulonglong2 bk = *reinterpret_cast<const ulonglong2*>(&bsm[i][k]);
#pragma unroll
                    for (int p = 0; p < 4; ++p) acc[h][p] = fma2_pk(bk.x, a[k][p], acc[h][p]);
#pragma unroll
                    for (int p = 0; p < 4; ++p) acc[h][p] = fma2_pk(bk.y, a[k + 1][p], acc[h][p]);
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t wv[4] = {w[h].x, w[h].y, w[h].z, w[h].w};
                uint32_t xo[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    if constexpr (FUSED) {
                        const float2 m = unpk2(fma2_pk(s2, acc[h][p], pk2(bf16_lo(wv[p]), bf16_hi(wv[p]))));
                        xo[p] = cvt_bf16x2(m.y, m.x);
                    } else {
                        // scalar: a paired product must not feed an add (see mul2_rn)
                        const float2 sp = unpk2(acc[h][p]);
                        xo[p] = cvt_bf16x2(__fadd_rn(bf16_hi(wv[p]), __fmul_rn(scale, sp.y)),
                                           __fadd_rn(bf16_lo(wv[p]), __fmul_rn(scale, sp.x)));
                    }
                }
                const bool keep = FULL || (colok && 2 * st + h < n);
                if constexpr (kNV) {
                    const int64_t e = erow + h * cols;
                    // every lane runs the codec (its block max is a pair shuffle); rows past
                    // the end repeat the last row and are not stored
                    Elems<uint16_t, 8> xe;
                    xe.v[0] = make_uint4(xo[0], xo[1], xo[2], xo[3]);
                    Fp4Lane o;
                    fp4_lane<true, true, QF_LORA8_TAB>(xe, s_t, six_st, o, yd, &s_tab[0]);
                    if (keep) {
                        if (T.y) *reinterpret_cast<uint4*>(T.y + e) = o.y;
                        if (T.codes) *reinterpret_cast<uint32_t*>(T.codes + (e >> 1)) = o.codes;
                        if (T.scales && (lane & 1) == 0) T.scales[e >> 4] = (uint8_t)o.scale;
                    }
                }
                if (kWritesMerged && keep)
                    *reinterpret_cast<uint4*>(yrow + h * cols) = make_uint4(xo[0], xo[1], xo[2], xo[3]);
                if (kFoldsAmax)
                    run = max_u16x2(max_u16x2(run, max_u16x2(xo[0] & 0x7FFF7FFFu, xo[1] & 0x7FFF7FFFu)),
                                    max_u16x2(xo[2] & 0x7FFF7FFFu, xo[3] & 0x7FFF7FFFu));
            }
            if (kWritesMerged) yrow += 2 * cols;
            if (kNV) erow += 2 * cols;
        }
        cp_async_wait<0>();
    };
    if (nrows == kLora8Rows && colok) {
        if (fused) unit(FullTile<true>{}, FullTile<true>{});
        else unit(FullTile<true>{}, FullTile<false>{});
    } else {
        if (fused) unit(FullTile<false>{}, FullTile<true>{});
        else unit(FullTile<false>{}, FullTile<false>{});
    }

    if (kFoldsAmax) {
        __shared__ uint32_t wmax[kLora8Threads / 32];
        run = bf16x2_max_bits(run);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) run = max(run, __shfl_xor_sync(kFull, run, o));
        if (lane == 0) wmax[wid] = run;
        __syncthreads();
        if (threadIdx.x == 0) {
            for (int w = 1; w < kLora8Threads / 32; ++w) run = max(run, wmax[w]);
            if (run != 0)
                atomicMax(reinterpret_cast<unsigned int*>(const_cast<float*>(P.group_amax)) + T.group,
                          run);
        }
    }
}

// ------------------------------------------------------------------ merged-weight amax
// k_lora_amax: the exact max |M| of a tie group's merged weights, M = BF16(W + s * acc),
// with the rank-r merge evaluated only where it can decide the result.
//
// Bounds.  With R_i = sum_k |b_ik| (FP32) and C_j = max_k |a_kj|, every term satisfies
// |b_ik a_kj| <= |b_ik| C_j, so |sum_k b_ik a_kj| <= R_i C_j.  The fused sum, the
// scaling, the add and the BF16 rounding each add at most one rounding (or, where the
// value is subnormal, an absolute error below 2^-133), so for
//   D_ij = K_i C_j + 2^-120 + |s| 2^-140,   K_i = |s| R_i (1 + 2^-6)
//   (D_ij = 0 when K_i or C_j is 0: every product is then an exact zero and M = W)
// every element satisfies
//   lb = (|W| - D_ij)(1 - 2^-7) - 2^-120  <=  |M|  <=  (|W| + D_ij)(1 + 2^-7) = ub,
// with the FP32 rounding of these expressions themselves inside the margins (2^-6 and
// 2^-7 against a few 2^-24).  An element whose ub is below a lower bound of the group's
// max |M| cannot be that max.  The lower bounds used: the lb of any element, and the
// exact |M| of any evaluated element, including the group's current amax (the output
// only ever receives exact values).
//
// Pass 1 reads the CTA's tile (kLoraAmaxRows rows x 1024 columns) and keeps, per row and
// lane, the max |W| of the lane's 32 elements; the CTA's best lb follows from it.  Its
// first row pair is requested before the prologue (the adapters' maxima) and every
// later pair one step ahead, so the tile's reads stay in flight.
// Pass 2 revisits only the (row, lane) pieces whose bound reaches that lower bound and
// re-reads their 32 elements (from L2); the elements whose own bound still reaches it go
// to a per-warp queue in shared memory, and the warp evaluates the queue 32 elements at
// a time, one per lane, with the merge kernel's arithmetic (each element's rank-r terms
// fetched 8 at a time).  The result is the max over the evaluated elements: exact, since
// the max element is always evaluated.
#ifndef QF_LORA_AMAX_ROWS
#define QF_LORA_AMAX_ROWS 128
#endif
constexpr int kLoraAmaxRows = QF_LORA_AMAX_ROWS;     // a multiple of 2 * kLoraThreads / 32
constexpr float kBoundUp = 1.0f + 0x1p-7f;
constexpr float kBoundDown = 1.0f - 0x1p-7f;
constexpr float kBoundWiden = 1.0f + 0x1p-6f;
constexpr float kBoundTiny = 0x1p-120f;

// |M| of element (i, j) as FP32: the merge of k_lora, one element at a time, with the
// terms' operands fetched 8 at a time (8 loads of B's row and 8 of A's column in flight
// together); the terms are still added one by one in increasing k.
__device__ __forceinline__ float lora_merged_mag(const LoraTensor& T, int64_t i, int64_t j,
                                                  float w) {
    const uint16_t* bp = T.b + i * T.rank;
    const uint16_t* ap = T.a + j;
    float acc = 0.0f;
#pragma unroll 1
    for (int k0 = 0; k0 < T.rank; k0 += 8) {
        float bv[8], av[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const bool ok = k0 + u < T.rank;
            bv[u] = ok ? bf16_lo(bp[k0 + u]) : 0.0f;
            av[u] = ok ? bf16_lo(ap[(int64_t)(k0 + u) * T.cols]) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (k0 + u < T.rank) acc = __fmaf_rn(bv[u], av[u], acc);
    }
    const uint32_t m = cvt_bf16x2(0.0f, __fadd_rn(w, __fmul_rn(T.scale, acc)));
    return __uint_as_float((m & 0x7FFFu) << 16);
}

__device__ __forceinline__ uint32_t max_abs_bf16x8(uint32_t m, uint4 v) {
    m = max_u16x2(m, v.x & 0x7FFF7FFFu);
    m = max_u16x2(m, v.y & 0x7FFF7FFFu);
    m = max_u16x2(m, v.z & 0x7FFF7FFFu);
    return max_u16x2(m, v.w & 0x7FFF7FFFu);
}

#ifndef QF_LORA_AMAX_LD
#define QF_LORA_AMAX_LD 0       // pass 1's loads of W (ld_stream form)
#endif
#ifndef QF_LORA_AMAX_MINB
#define QF_LORA_AMAX_MINB 3     // 3 CTAs per SM (80 registers): 61.5 us against 77.9 at 2
#endif
template <int MAXT>
__global__ void __launch_bounds__(kLoraThreads, QF_LORA_AMAX_MINB) k_lora_amax(const __grid_constant__ LoraTable<MAXT> P) {
    constexpr int kWarps = kLoraThreads / 32;
    constexpr int kRpw = kLoraAmaxRows / kWarps;         // rows per warp, read two at a time
    constexpr int kChunks = kLoraCols / 8;                // 16-byte column chunks per tile row
    static_assert(kLoraAmaxRows % (2 * kWarps) == 0, "row pairs per warp");
    static_assert(kLoraThreads >= 2 * kChunks && kLoraThreads >= kLoraAmaxRows, "prologue shape");
    __shared__ float s_k[kLoraAmaxRows];                  // K_i
    __shared__ float s_c[kLoraCols];                      // C_j
    __shared__ uint4 s_cpart[2][kChunks];                 // per-chunk |a| maxima, two k halves
    __shared__ uint32_t s_lb, s_best;
    constexpr int kQueue = 64;                            // pass-2 queue entries per warp
    __shared__ uint2 s_q[kWarps][kQueue];                 // (row << 16 | column, W bits)
    __shared__ uint32_t s_qn[kWarps];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (blockIdx.x >= P.total_units) return;
    const LoraTensor& T = P.t[lora_locate(P, blockIdx.x)];
    const int64_t local = blockIdx.x - T.unit_begin;
    const int64_t r0 = (local / T.col_groups) * kLoraAmaxRows;
    const int64_t c_base = (local % T.col_groups) * kLoraCols;
    const int nrows = (int)min(T.rows - r0, (int64_t)kLoraAmaxRows);
    const int ncols = (int)min(T.cols - c_base, (int64_t)kLoraCols);   // a multiple of 16
    const int nchunks = ncols / 8;
    const int64_t cols = T.cols;
    const int rank = T.rank;
    const float sabs = fabsf(T.scale);
    const float tiny = __fadd_rn(kBoundTiny, __fmul_rn(sabs, 0x1p-140f));
    unsigned int* gamax = reinterpret_cast<unsigned int*>(const_cast<float*>(P.group_amax)) + T.group;
    const uint16_t* wlane = T.w + r0 * cols + c_base + 8 * lane;
    // pass 1's reads, a row pair (eight 16-byte loads per lane) per step: rows
    // wid + kWarps t and wid + kWarps (t + 1); the first pair is requested now
    auto load_pair = [&](int t, uint4 (&v)[2][4]) {
        const int i0 = wid + kWarps * t;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                v[h][q] = (i0 + h * kWarps < nrows && 256 * q + 8 * lane < ncols)
                              ? ld_stream<QF_LORA_AMAX_LD>(wlane + (i0 + h * kWarps) * cols + 256 * q)
                              : make_uint4(0, 0, 0, 0);
    };
    uint4 vbuf[2][2][4];
    load_pair(0, vbuf[0]);
    if (lane == 0) s_qn[wid] = 0u;

    // ---- prologue: C_j (16-byte loads of A, k split over two threads per chunk), K_i,
    // and the group's amax so far
    {
        const int c = threadIdx.x >> 1, h = threadIdx.x & 1;
        if (c < nchunks) {
            const uint16_t* ap = T.a + c_base + 8 * c;
            uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
#pragma unroll 4
            for (int k = h; k < rank; k += 2) {
                const uint4 v = ld_stream<1>(ap + k * cols);
                m0 = max_u16x2(m0, v.x & 0x7FFF7FFFu);
                m1 = max_u16x2(m1, v.y & 0x7FFF7FFFu);
                m2 = max_u16x2(m2, v.z & 0x7FFF7FFFu);
                m3 = max_u16x2(m3, v.w & 0x7FFF7FFFu);
            }
            s_cpart[h][c] = make_uint4(m0, m1, m2, m3);
        }
    }
    if (threadIdx.x < nrows) {
        const uint16_t* bp = T.b + (r0 + threadIdx.x) * rank;
        float r = 0.0f;
#pragma unroll 8
        for (int k = 0; k < rank; ++k) r = __fadd_rn(r, fabsf(bf16_lo(bp[k])));
        s_k[threadIdx.x] = __fmul_rn(__fmul_rn(sabs, r), kBoundWiden);
    }
    if (threadIdx.x == 0) {
        s_best = *reinterpret_cast<volatile unsigned int*>(gamax);
        s_lb = 0u;
    }
    __syncthreads();
    if (threadIdx.x < nchunks) {
        const uint4 p0 = s_cpart[0][threadIdx.x], p1 = s_cpart[1][threadIdx.x];
        const uint32_t m[4] = {max_u16x2(p0.x, p1.x), max_u16x2(p0.y, p1.y),
                               max_u16x2(p0.z, p1.z), max_u16x2(p0.w, p1.w)};
#pragma unroll
        for (int e = 0; e < 8; ++e)
            s_c[8 * threadIdx.x + e] = __uint_as_float(((m[e >> 1] >> (16 * (e & 1))) & 0xFFFFu) << 16);
    }
    __syncthreads();

    // this lane's columns: c_base + 256 q + 8 lane + e, q < 4, e < 8
    float cmax = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q)
        if (256 * q + 8 * lane < ncols)
#pragma unroll
            for (int e = 0; e < 8; ++e) cmax = fmaxf(cmax, s_c[256 * q + 8 * lane + e]);
    auto dbound = [&](float k, float c) {
        return (k > 0.0f && c > 0.0f) ? __fadd_rn(__fmul_rn(k, c), tiny) : 0.0f;
    };

    // ---- pass 1: max |W| per (row, lane), a row pair per step with the next pair's
    // loads in flight; the best lower bound
    float mrow[kRpw];
    float lb_best = 0.0f;
#pragma unroll
    for (int t = 0; t < kRpw; t += 2) {
        const int i0 = wid + kWarps * t, i1 = i0 + kWarps;
        if (t + 2 < kRpw) load_pair(t + 2, vbuf[((t >> 1) + 1) & 1]);
        const uint4 (&v)[2][4] = vbuf[(t >> 1) & 1];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t m = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) m = max_abs_bf16x8(m, v[h][q]);
            const int i = h ? i1 : i0;
            mrow[t + h] = __uint_as_float(bf16x2_max_bits(m));
            if (i < nrows) {
                const float lb = __fsub_rn(__fmul_rn(__fsub_rn(mrow[t + h], dbound(s_k[i], cmax)),
                                                     kBoundDown), kBoundTiny);
                lb_best = fmaxf(lb_best, lb);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lb_best = fmaxf(lb_best, __shfl_xor_sync(kFull, lb_best, o));
    if (lane == 0 && lb_best > 0.0f) atomicMax(&s_lb, __float_as_uint(lb_best));
    __syncthreads();

    // ---- pass 2: exact merges where the bound reaches the lower bound.  The (row, lane)
    // pieces to revisit are marked first (unrolled, so mrow stays in registers); the
    // rare revisits then run as plain loops.
    float best = __uint_as_float(s_best);                 // exact: the group's amax so far
    const float L = fmaxf(__uint_as_float(s_lb), best);
    uint32_t cand = 0;
#pragma unroll
    for (int t = 0; t < kRpw; ++t) {
        const int i = wid + kWarps * t;
        const float rowub = __fmul_rn(__fadd_rn(mrow[t], dbound(i < nrows ? s_k[i] : 0.0f, cmax)),
                                      kBoundUp);
        if (i < nrows && rowub >= L && rowub > best) cand |= 1u << t;
    }
    // the elements of those pieces whose own bound reaches L, into the warp's queue (an
    // element past its capacity is evaluated on the spot)
#pragma unroll 1
    while (cand) {
        const int t = __ffs(cand) - 1;
        cand &= cand - 1;
        const int i = wid + kWarps * t;
        const float ki = s_k[i];
        uint4 vq[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            vq[q] = 256 * q + 8 * lane < ncols ? ld_stream<1>(wlane + i * cols + 256 * q)
                                               : make_uint4(0, 0, 0, 0);
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
            const int c0 = 256 * q + 8 * lane;
            if (c0 >= ncols) continue;
            const uint64_t lo = vq[q].x | (uint64_t)vq[q].y << 32;
            const uint64_t hi = vq[q].z | (uint64_t)vq[q].w << 32;
#pragma unroll 1
            for (int e = 0; e < 8; ++e) {
                const uint32_t wb = (uint32_t)(((e < 4 ? lo : hi) >> (16 * (e & 3))) & 0xFFFFu);
                const float x = __uint_as_float((wb & 0x7FFFu) << 16);
                const float ub = __fmul_rn(__fadd_rn(x, dbound(ki, s_c[c0 + e])), kBoundUp);
                if (ub >= L && ub > best) {
                    const uint32_t pos = atomicAdd(&s_qn[wid], 1u);
                    if (pos < (uint32_t)kQueue)
                        s_q[wid][pos] = make_uint2((uint32_t)i << 16 | (uint32_t)(c0 + e), wb);
                    else
                        best = fmaxf(best, lora_merged_mag(T, r0 + i, c_base + c0 + e,
                                                            __uint_as_float(wb << 16)));
                }
            }
        }
    }
    __syncwarp();
    // the queue, 32 elements at a time, each skipped once the warp's best exceeds its bound
    const int nq = (int)min(s_qn[wid], (uint32_t)kQueue);
#pragma unroll 1
    for (int b0 = 0; b0 < nq; b0 += 32) {
        float wbest = best;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wbest = fmaxf(wbest, __shfl_xor_sync(kFull, wbest, o));
        if (b0 + lane < nq) {
            const uint2 q = s_q[wid][b0 + lane];
            const int i = (int)(q.x >> 16), c = (int)(q.x & 0xFFFFu);
            const float x = __uint_as_float((q.y & 0x7FFFu) << 16);
            const float ub = __fmul_rn(__fadd_rn(x, dbound(s_k[i], s_c[c])), kBoundUp);
            if (ub > wbest)
                best = fmaxf(best, lora_merged_mag(T, r0 + i, c_base + c,
                                                    __uint_as_float(q.y << 16)));
        }
    }
    // ---- the CTA's best exact value into the group's amax
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = fmaxf(best, __shfl_xor_sync(kFull, best, o));
    if (lane == 0 && best > 0.0f) atomicMax(gamax, __float_as_uint(best));
}

}  // namespace qf
