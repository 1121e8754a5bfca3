// qf_oneshot.cuh -- NVFP4 tie-group amax and fake-quant + pack in ONE launch, for calls
// whose inputs fit in L2 (sm_100a: 126 MB).
//
// NVFP4 needs the FP32 tensor scale s_t = amax_g / 2688 of a whole tie group before
// any block can be encoded (QATFactory project page, Method, "Numerics": one
// tensor-level scale shared by the fused projections), so the plain path is two
// launches that both read the input from HBM.  For an input that fits in L2 this
// kernel runs both phases in one cooperative launch:
//   phase 1  every CTA reads its units from HBM and folds max |x| into per-group
//            slots of a device workspace (atomicMax on the FP32 bits, after a
//            CTA-level combine);
//   barrier  a grid-wide arrive counter; all CTAs are co-resident (cooperative launch),
//            and the wait is bounded: after kOneshotSpinLimit polls the CTA sets the
//            workspace's error word and skips phase 2 (its outputs stay unwritten);
//   phase 2  every CTA re-reads the same units -- now L2 hits -- and encodes them
//            exactly as k_nv does.
// Every CTA departs through a second counter, whether it passed the barrier or gave
// up; the last one out resets the slots and both counters, so the workspace is zero
// again after every call, a timed-out one included.  The error word is sticky: it
// stays set until the host clears it (qf_workspace_check), and a call that finds it
// set at entry does no work at all, so no later call can encode from a partial amax.
//
// Every fold of the amax (slots, the tracked running value) takes the max of the FP32
// bit patterns as unsigned integers, as k_amax does: for values >= +0 that is the
// float max, and a NaN running value stays NaN, on both paths of the call alike.
//
// Workspace layout (32-bit words): [0] error flags, [1] reserved (0), [2] arrive
// count, [3] depart count, [4 + g] group g's running max |x| as FP32 bits.
#pragma once

#include "qf_device.cuh"

namespace qf {

constexpr int kOneshotHeaderWords = 4;
constexpr uint32_t kOneshotSpinLimit = 1u << 22;    // polls, ~256 ns apart: about a second
constexpr uint32_t kOneshotErrTimeout = 1u;
constexpr int kOneshotErrWord = 0, kOneshotArriveWord = 2, kOneshotDepartWord = 3;
#ifndef QF_ONESHOT_THREADS
#define QF_ONESHOT_THREADS 256
#endif
#ifndef QF_ONESHOT_MINB
#define QF_ONESHOT_MINB 1       // minimum resident CTAs per SM asked of the register allocator
#endif
#ifndef QF_ONESHOT_L2_DIV
#define QF_ONESHOT_L2_DIV 3     // single-launch path when all input bytes <= L2 size / this
#endif

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// ---- the parts both one-launch kernels share

// A sticky error left by an earlier call on this workspace: the CTA does no work.
__device__ __forceinline__ bool oneshot_skip(const uint32_t* ws) {
    __shared__ int s_skip;
    if (threadIdx.x == 0) s_skip = ld_relaxed_gpu(ws + kOneshotErrWord) != 0u;
    __syncthreads();
    const bool skip = s_skip;
    __syncthreads();
    return skip;
}

// Combine the warps' last (group, max) pairs in the CTA; one atomicMax per CTA and group.
template <int THREADS>
__device__ __forceinline__ void oneshot_fold(uint32_t* slot, int g, uint32_t a) {
    constexpr int kWarps = THREADS / 32;
    __shared__ int wgrp[kWarps];
    __shared__ uint32_t wmax[kWarps];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0) {
        wgrp[wid] = g;
        wmax[wid] = a;
    }
    __syncthreads();
    if (threadIdx.x < kWarps) {
        const int w = threadIdx.x, gw = wgrp[w];
        bool first = gw >= 0;
        uint32_t m = wmax[w];
        for (int o = 0; o < kWarps; ++o) {
            if (wgrp[o] != gw) continue;
            if (o < w) first = false;
            m = max(m, wmax[o]);
        }
        if (first) atomicMax(slot + gw, m);
    }
    __syncthreads();
}

// The bounded grid barrier; returns whether this CTA may go on to phase 2.
__device__ __forceinline__ bool oneshot_barrier(uint32_t* ws, bool skip, uint32_t test_polls) {
    __shared__ int s_go;
    if (threadIdx.x == 0) {
        __threadfence();                                    // this CTA's slot updates first
        atomicAdd(ws + kOneshotArriveWord, 1u);
        bool done = false;
        if (!skip) {
            const uint32_t target = gridDim.x + (test_polls ? 1u : 0u);
            const uint32_t limit = test_polls ? test_polls : kOneshotSpinLimit;
            uint32_t polls = 0;
            done = ld_acquire_gpu(ws + kOneshotArriveWord) >= target;
            while (!done && ++polls < limit) {
                __nanosleep(256);
                done = ld_acquire_gpu(ws + kOneshotArriveWord) >= target;
            }
            if (!done) atomicOr(ws + kOneshotErrWord, kOneshotErrTimeout);
        }
        s_go = done;
    }
    __syncthreads();
    return s_go;
}

// The effective amax of a group: this call's max, folded with the running value when
// one is kept (FP32 bit patterns as unsigned integers, as k_amax folds them).
template <int MAXT>
__device__ __forceinline__ float oneshot_eff_amax(const Table<MAXT>& P, const uint32_t* slot,
                                                  int grp) {
    uint32_t a = ld_relaxed_gpu(slot + grp);
    if (P.tracked) a = max(a, __float_as_uint(P.tracked[grp]));
    return __uint_as_float(a);
}

// CTA 0 writes the group statistics: this call's amax, the running amax, s_t.
template <int MAXT, int THREADS>
__device__ __forceinline__ void oneshot_stats(const Table<MAXT>& P, const uint32_t* slot) {
    if (blockIdx.x != 0) return;
    for (int q = threadIdx.x; q < P.n_groups; q += THREADS) {
        const float cur = __uint_as_float(ld_relaxed_gpu(slot + q));
        const float e = oneshot_eff_amax(P, slot, q);
        const_cast<float*>(P.group_amax)[q] = cur;
        if (P.tracked) P.tracked[q] = e;
        if (P.group_scale_out) P.group_scale_out[q] = nv_tensor_scale(e);
    }
}

// Every CTA departs, whether it passed the barrier or gave up; the last one out leaves
// the slots and counters zeroed for the next call.
template <int THREADS>
__device__ __forceinline__ void oneshot_depart(uint32_t* ws, int n_groups) {
    __shared__ int s_last;
    uint32_t* slot = ws + kOneshotHeaderWords;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = atomicAdd(ws + kOneshotDepartWord, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (s_last) {
        __threadfence();
        for (int q = threadIdx.x; q < n_groups; q += THREADS) slot[q] = 0u;
        if (threadIdx.x == 0) {
            ws[kOneshotArriveWord] = 0u;
            ws[kOneshotDepartWord] = 0u;
        }
    }
}

// ---- k_nv_oneshot: the second pass re-reads x from L2
// P.group_amax: output, this call's tie-group amax.  P.tracked (nullable): running
// amax, max-accumulated in place; when given, s_t comes from the updated running
// value (the activation reading), otherwise from this call's amax.
// P.group_scale_out (nullable): s_t per group.
// test_polls: 0 in normal use.  N > 0 makes the barrier wait for one CTA more than the
// grid holds, polling at most N times, so that every CTA gives up: the timeout path
// runs with every CTA present and no fault.
template <typename XT, int U, int MAXT, int THREADS>
__global__ void __launch_bounds__(THREADS, QF_ONESHOT_MINB)
    k_nv_oneshot(const __grid_constant__ Table<MAXT> P, uint32_t* __restrict__ ws,
                 uint32_t test_polls) {
    constexpr int kWarps = THREADS / 32;
    constexpr int kUnit = 512 * U;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t warp = int64_t(blockIdx.x) * kWarps + wid;
    const int64_t nwarps = int64_t(gridDim.x) * kWarps;
    uint32_t* slot = ws + kOneshotHeaderWords;
    const bool skip = oneshot_skip(ws);

    // ---- phase 1: max |x| per tie group over this warp's units
    int ti = warp < P.total_units && !skip ? locate_tensor(P, warp) : 0;
    int g = -1;
    uint32_t run = 0;
    auto warp_max = [&]() {
        uint32_t a = run;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(kFull, a, o));
        return a;
    };
    for (int64_t u = skip ? P.total_units : warp; u < P.total_units; u += nwarps) {
        ti = find_tensor(P, ti, u);
        const DevTensor& T = P.t[ti];
        if (T.group != g) {
            const uint32_t a = warp_max();
            if (lane == 0 && g >= 0) atomicMax(slot + g, a);
            run = 0;
            g = T.group;
        }
        Elems<XT, 16> v[U];
        nv_load_unit<XT, U, 1>(T, (u - T.unit_begin) * kUnit, lane, v);
#pragma unroll
        for (int s = 0; s < U; ++s) run = max(run, v[s].amax_bits());
    }
    oneshot_fold<THREADS>(slot, g, warp_max());

    const bool go = oneshot_barrier(ws, skip, test_polls);   // false: outputs left unwritten
    if (go) oneshot_stats<MAXT, THREADS>(P, slot);

    // ---- phase 2: encode the same units (their lines are in L2 now)
    if (go && warp < P.total_units) {
        ti = locate_tensor(P, warp);
        int cur_t = -1;
        float s_t = 0.0f, six_st = 0.0f;
        for (int64_t u = warp; u < P.total_units; u += nwarps) {
            ti = find_tensor(P, ti, u);
            const DevTensor& T = P.t[ti];
            if (ti != cur_t) {
                s_t = nv_tensor_scale(oneshot_eff_amax(P, slot, T.group));
                six_st = __fmul_rn(6.0f, s_t);
                cur_t = ti;
            }
            const int64_t e0 = (u - T.unit_begin) * kUnit;
            Elems<XT, 16> v[U];
            nv_load_unit<XT, U, 1>(T, e0, lane, v);
            nv_encode_unit<XT, U>(T, e0, lane, v, s_t, six_st);
        }
    }
    oneshot_depart<THREADS>(ws, P.n_groups);
}

}  // namespace qf
