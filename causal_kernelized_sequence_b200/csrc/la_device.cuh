// la_device.cuh -- device helpers shared by the libla kernels: element I/O,
// the two feature maps, and the per-device status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/la.h"

namespace la {

// Status word written by kernels that detect an error on the device (a
// bounded wait that ran out, a failed check).  Read and cleared by
// la_get_device_status.  Bits: 1 = timeout, 2 = device check.  The library
// is built as one translation unit, so this definition is unique.
__device__ unsigned int g_status;

constexpr unsigned int kStatusTimeout = 1u;
constexpr unsigned int kStatusCheck = 2u;

__device__ __forceinline__ void report(unsigned int bit) { atomicOr(&g_status, bit); }

// ------------------------------------------------------------ element I/O
template <typename T> __device__ __forceinline__ float ld(const T *p);
template <> __device__ __forceinline__ float ld<float>(const float *p) { return *p; }
template <> __device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16 *p)
{
    return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ void st(T *p, float x);
template <> __device__ __forceinline__ void st<float>(float *p, float x) { *p = x; }
template <> __device__ __forceinline__ void st<__nv_bfloat16>(__nv_bfloat16 *p, float x)
{
    *p = __float2bfloat16_rn(x);
}

// ------------------------------------------------------------ feature maps
// Constants of the Taylor map, computed on the host in double precision and
// rounded once: inv_c1 = 1/dqk^(1/4), inv_c2 = 1/(sqrt(2) sqrt(dqk)),
// inv_c3 = 1/sqrt(dqk) (the folded map's pair features).
struct FmapParams {
    int fmap;   // LA_FMAP_ELU1, LA_FMAP_TAYLOR2 or LA_FMAP_TAYLOR2_SYM
    int dqk;
    int F;
    float inv_c1;
    float inv_c2;
    float inv_c3;
};

// elu(x)+1 with alpha = 1 ("Transformers are RNNs").
__device__ __forceinline__ float elu1(float x) { return x > 0.f ? x + 1.f : expf(x); }
__device__ __forceinline__ float elu1_grad(float x) { return x > 0.f ? 1.f : expf(x); }

// Pair number p of the folded Taylor map's cross block -> (a, b), a < b,
// pairs in row-major order (0,1), (0,2), ..., (1,2), ...
__host__ __device__ __forceinline__ void sym_pair(int p, int d, int &a, int &b)
{
    a = 0;
    while (p >= d - 1 - a) {
        p -= d - 1 - a;
        ++a;
    }
    b = a + 1 + p;
}

// Inverse of sym_pair for a < b.
__host__ __device__ __forceinline__ int sym_pair_index(int a, int b, int d)
{
    return a * d - a * (a + 1) / 2 + (b - a - 1);
}

// Feature f of phi(x) for a vector x held in shared/local memory.
// TAYLOR2:     [1 | x_a * inv_c1 | x_a x_b * inv_c2 (row-major a, b)].
// TAYLOR2_SYM: [1 | x_a * inv_c1 | x_a^2 * inv_c2 | x_a x_b * inv_c3 (a < b)].
__device__ __forceinline__ float phi_feature(const FmapParams &fp, const float *x, int f)
{
    if (fp.fmap == LA_FMAP_ELU1) return elu1(x[f]);
    if (f == 0) return 1.f;
    if (f <= fp.dqk) return x[f - 1] * fp.inv_c1;
    const int idx = f - 1 - fp.dqk;
    if (fp.fmap == LA_FMAP_TAYLOR2_SYM) {
        if (idx < fp.dqk) return x[idx] * x[idx] * fp.inv_c2;
        int a, b;
        sym_pair(idx - fp.dqk, fp.dqk, a, b);
        return x[a] * x[b] * fp.inv_c3;
    }
    const int a = idx / fp.dqk, b = idx - a * fp.dqk;
    return x[a] * x[b] * fp.inv_c2;
}

// dx_c = sum_f dphi_f d phi_f / d x_c  for one vector (c = component).
__device__ __forceinline__ float phi_vjp_component(const FmapParams &fp, const float *x,
                                                   const float *dphi, int c)
{
    if (fp.fmap == LA_FMAP_ELU1) return dphi[c] * elu1_grad(x[c]);
    const int d = fp.dqk;
    if (fp.fmap == LA_FMAP_TAYLOR2_SYM) {
        // d/dx_c: x_c^2 inv_c2 -> 2 x_c inv_c2;  x_a x_b inv_c3 -> x_b inv_c3 (c = a) or x_a inv_c3 (c = b)
        const float *dp = dphi + 1 + 2 * d;
        float t = 0.f;
        for (int b = 0; b < d; ++b)
            if (b != c) t = fmaf(dp[b < c ? sym_pair_index(b, c, d) : sym_pair_index(c, b, d)], x[b], t);
        const float s = fmaf(dphi[1 + d + c] * 2.f * x[c], fp.inv_c2, dphi[1 + c] * fp.inv_c1);
        return fmaf(t, fp.inv_c3, s);
    }
    float s = dphi[1 + c] * fp.inv_c1;
    float t = 0.f;
    for (int b = 0; b < d; ++b)
        t = fmaf(dphi[1 + d + c * d + b] + dphi[1 + d + b * d + c], x[b], t);
    return fmaf(t, fp.inv_c2, s);
}

}  // namespace la
