// la_decode.cuh -- bandwidth-bound recurrent decode step.
//
// BASED page, Knowl 3 recurrent form and Knowl 5 generation kernel: for each
// head, S += phi(k) v^T, z += phi(k), y = phi(q) S / phi(q).z on the updated
// state; with a forget gate a = exp(g) per head, S = a S + phi(k) v^T and
// z = a z + phi(k) (the gated update of the 'Transformers are RNNs'
// discussion page).  The state (F x DV fp32 plus F fp32) is read once and written once
// per call; everything else is noise, so the kernel is organised around HBM:
//
//  - one 256-thread block per head; thread (r0, c4) owns the float4 column
//    group c4 of rows r0, r0 + RPP, r0 + 2 RPP, ... (RPP = 256 / (DV/4)), so
//    each warp moves whole 128-byte lines with 16-byte loads and stores;
//  - MINB blocks per SM: 2 for the 273-row Taylor state, more for states of
//    at most MAXP = 10 passes (the 153-row folded state), whose blocks are
//    shorter, so that more of them keep loads in flight;
//  - every state load of a batch of up to MAXP row passes is issued before
//    the block computes phi(q), phi(k) (the feature-map prologue overlaps the
//    first DRAM round trip) and before any of them is consumed, keeping
//    MAXP x 16 bytes in flight per thread;
//  - the state is streamed (evict-first loads and stores: it is not reused
//    within the step and exceeds L2 across heads);
//  - the numerator is reduced across row groups with shuffles, then across
//    warps in shared memory, in a fixed order (deterministic).
#pragma once

#include "la_device.cuh"
#include "sm100.cuh"

namespace la {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeMaxF = 288;

template <typename T, int DV, int MAXP, int MINB>
__global__ void __launch_bounds__(kDecodeThreads, MINB)
decode_vec_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                  T *__restrict__ y, float *__restrict__ S, float *__restrict__ z, FmapParams fp,
                  const float *__restrict__ logdecay)
{
    constexpr int CPR = DV / 4;                  // float4 groups per state row
    constexpr int RPP = kDecodeThreads / CPR;    // rows per pass
    constexpr int NW = kDecodeThreads / 32;
    static_assert(CPR >= 1 && (32 % CPR == 0 || CPR % 32 == 0), "row split must align to warps");

    __shared__ float pq[kDecodeMaxF], pk[kDecodeMaxF];
    __shared__ float xq[128], xk[128];
    __shared__ __align__(16) float vv[DV];
    __shared__ float red[NW][DV];
    __shared__ float dred[NW];

    // Launched as a programmatic dependent: the previous step's state and
    // outputs are complete and visible once this returns; the next step's
    // blocks may then take the SMs this grid leaves.
    sm100::grid_dependency_wait();
    sm100::launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c4 = tid % CPR, r0 = tid / CPR;
    const int F = fp.F, dqk = fp.dqk;
    const size_t bh = blockIdx.x;
    float4 *Sb = reinterpret_cast<float4 *>(S + bh * (size_t)F * DV);
    float *zb = z + bh * (size_t)F;
    const int passes = (F + RPP - 1) / RPP;

    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 vc = acc;
    float4 sreg[MAXP];
    // z entries of this thread (F <= kDecodeMaxF < 2 x 256), loaded with the
    // first batch of state rows rather than after the last one.
    static_assert(kDecodeMaxF <= 2 * kDecodeThreads, "two z entries per thread");
    const float z0 = tid < F ? __ldcs(zb + tid) : 0.f;
    const float z1 = tid + kDecodeThreads < F ? __ldcs(zb + tid + kDecodeThreads) : 0.f;
    // gated form: the head's forget gate a = exp(g) scales the state first (1 ungated)
    const float gate = logdecay ? expf(logdecay[bh]) : 1.f;
    for (int p0 = 0; p0 < passes; p0 += MAXP) {
#pragma unroll
        for (int b = 0; b < MAXP; ++b) {
            const int f = r0 + (p0 + b) * RPP;
            if (p0 + b < passes && f < F) sreg[b] = __ldcs(Sb + (size_t)f * CPR + c4);
        }
        if (p0 == 0) {
            // Feature maps of this head's query and key, and the value row.
            for (int i = tid; i < dqk; i += kDecodeThreads) {
                xq[i] = ld(q + bh * dqk + i);
                xk[i] = ld(k + bh * dqk + i);
            }
            for (int i = tid; i < DV; i += kDecodeThreads) vv[i] = ld(v + bh * DV + i);
            __syncthreads();
            for (int f = tid; f < F; f += kDecodeThreads) {
                pq[f] = phi_feature(fp, xq, f);
                pk[f] = phi_feature(fp, xk, f);
            }
            __syncthreads();
            vc = reinterpret_cast<const float4 *>(vv)[c4];
        }
#pragma unroll
        for (int b = 0; b < MAXP; ++b) {
            const int f = r0 + (p0 + b) * RPP;
            if (p0 + b < passes && f < F) {
                const float a = pk[f], w = pq[f];
                float4 s = sreg[b];
                s.x = fmaf(a, vc.x, gate * s.x);
                s.y = fmaf(a, vc.y, gate * s.y);
                s.z = fmaf(a, vc.z, gate * s.z);
                s.w = fmaf(a, vc.w, gate * s.w);
                __stcs(Sb + (size_t)f * CPR + c4, s);
                acc.x = fmaf(w, s.x, acc.x);
                acc.y = fmaf(w, s.y, acc.y);
                acc.z = fmaf(w, s.z, acc.z);
                acc.w = fmaf(w, s.w, acc.w);
            }
        }
    }
    // z update and the denominator phi(q).z (z rows are 4-byte aligned only).
    float dacc = 0.f;
    if (tid < F) {
        const float zz = fmaf(gate, z0, pk[tid]);
        __stcs(zb + tid, zz);
        dacc = pq[tid] * zz;
    }
    if (tid + kDecodeThreads < F) {
        const float zz = fmaf(gate, z1, pk[tid + kDecodeThreads]);
        __stcs(zb + tid + kDecodeThreads, zz);
        dacc = fmaf(pq[tid + kDecodeThreads], zz, dacc);
    }
    // Numerator: reduce row groups inside the warp, then across warps.
    if (CPR < 32) {
#pragma unroll
        for (int off = CPR; off < 32; off <<= 1) {
            acc.x += __shfl_xor_sync(0xffffffffu, acc.x, off);
            acc.y += __shfl_xor_sync(0xffffffffu, acc.y, off);
            acc.z += __shfl_xor_sync(0xffffffffu, acc.z, off);
            acc.w += __shfl_xor_sync(0xffffffffu, acc.w, off);
        }
    }
    if (lane < CPR || CPR >= 32) {
        const int col = 4 * c4;
        red[warp][col] = acc.x;
        red[warp][col + 1] = acc.y;
        red[warp][col + 2] = acc.z;
        red[warp][col + 3] = acc.w;
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) dacc += __shfl_xor_sync(0xffffffffu, dacc, off);
    if (lane == 0) dred[warp] = dacc;
    __syncthreads();
    if (tid < DV) {
        float den = 0.f, num = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            den += dred[w];
            num += red[w][tid];
        }
        st(y + bh * DV + tid, num / den);
    }
}

}  // namespace la
