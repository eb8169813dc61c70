// la_simt.cuh -- exact fp32 CUDA-core kernels for every entry point.
//
// These kernels compute in fp32 with plain FMA (no tensor cores, no TF32),
// one thread block per (batch, head) slice, walking the sequence in chunks of
// C tokens.  They are the path for fp32 I/O (where a 1e-5 relative error
// rules out bf16/TF32 tensor-core operands) and for the sizes the
// tensor-core kernels do not cover.  Everything lives in shared memory:
//
//   forward  (BASED page, Knowl 3 parallel form, chunked as in Knowl 5):
//     per chunk, A_ij = phi(q_i).phi(k_j) for j <= i inside the chunk,
//     num_i = sum_j A_ij v_j + phi(q_i) S,  den_i = sum_j A_ij + phi(q_i).z,
//     y_i = num_i / den_i, then S += phi(K_c)^T V_c, z += sum_j phi(k_j).
//   backward (derivative of the same form; see la.h):
//     forward-order pass for dq, reverse-order pass of R, r for dk, dv.
//   decode   (Knowl 3 recurrent form): S += phi(k) v^T, z += phi(k),
//     y = phi(q) S / phi(q).z on the updated state.
// The forward also takes a start state, packed sequences (a block per
// (sequence, head) of a [H, T, *] batch cut by cu_seqlens) and the gated form
// S_t = exp(g_t) S_{t-1} + phi(k_t) v_t^T.  Gated, every decay factor is the
// exponential of a plain sum of gates (a prefix, a suffix or a pair range),
// never a difference of prefix sums, so g = -inf gives exact zeros and no
// inf - inf.  The gated backward adds the gate gradient
// dL/dg_l = -sum_{j>=l} phi(k_j) . dL/dphi(k_j), summed in double.
#pragma once

#include "la_device.cuh"

namespace la {

constexpr int kSimtThreads = 256;

// Row strides padded to an odd number of floats so that column walks across
// a warp hit 32 different banks.
__host__ __device__ inline int odd_stride(int n) { return n | 1; }

struct SimtFwdSmem {
    int C, FS, DS;
    size_t floats(int F, int dqk, int dv) const
    {
        return (size_t)F * DS + F + 2 * (size_t)C * dqk + 2 * (size_t)C * FS + (size_t)C * dv +
               (size_t)C * C + 4 * (size_t)C;
    }
};

inline SimtFwdSmem simt_fwd_layout(int C, int F, int dv)
{
    return SimtFwdSmem{C, odd_stride(F), odd_stride(dv)};
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
fwd_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                T *__restrict__ o, const float *__restrict__ s_in, const float *__restrict__ z_in,
                float *__restrict__ s_out, float *__restrict__ z_out,
                float *__restrict__ den_out, int N, int dv, FmapParams fp, SimtFwdSmem L,
                const int *__restrict__ cu = nullptr, int H = 0, int T_total = 0,
                const float *__restrict__ logdecay = nullptr)
{
    extern __shared__ float sm[];
    const int F = fp.F, dqk = fp.dqk, C = L.C, FS = L.FS, DS = L.DS;
    float *S = sm;                      // [F][DS]
    float *z = S + (size_t)F * DS;      // [F]
    float *xq = z + F;                  // [C][dqk]
    float *xk = xq + C * dqk;           // [C][dqk]
    float *pq = xk + C * dqk;           // [C][FS]
    float *pk = pq + (size_t)C * FS;    // [C][FS]
    float *vs = pk + (size_t)C * FS;    // [C][dv]
    float *A = vs + C * dv;             // [C][C]
    float *den = A + C * C;             // [C]
    float *cum = den + C;               // [C]  gated form: L_i = g_{t0} + ... + g_{t0+i}
    float *wk = cum + C;                // [C]  exp(g_{t0+j+1} + ... + g_last): key j's weight in the state update
    float *graw = wk + C;               // [C]  the chunk's gates g_{t0+j}

    const int tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nwarps = nt >> 5;
    const size_t bh = blockIdx.x;   // the state slice
    // token rows of this slice: bh*N.. of [BH, N, *], or for packed sequences
    // (cu != null; slice = (n, h)) h*T_total + cu[n] .. of [H, T_total, *]
    size_t row0 = bh * N;
    if (cu) {
        const int n = (int)bh / H, h = (int)bh - n * H;
        const int a = cu[n], b = cu[n + 1];
        if (a < 0 || b < a || b > T_total || b - a > N) {   // N: the caller's max_seqlen
            if (tid == 0) report(kStatusCheck);
            return;
        }
        N = b - a;
        row0 = (size_t)h * T_total + a;
    }
    const T *qb = q + row0 * dqk;
    const T *kb = k + row0 * dqk;
    const T *vb = v + row0 * dv;
    T *ob = o + row0 * dv;

    // state entering the sequence: zero, or the given (s_in, z_in)
    for (int i = tid; i < F * DS; i += nt) {
        const int f = i / DS, c = i - f * DS;
        S[i] = (s_in && c < dv) ? s_in[bh * F * dv + (size_t)f * dv + c] : 0.f;
    }
    for (int i = tid; i < F; i += nt) z[i] = z_in ? z_in[bh * F + i] : 0.f;

    for (int t0 = 0; t0 < N; t0 += C) {
        const int Lc = min(C, N - t0);
        __syncthreads();
        for (int i = tid; i < Lc * dqk; i += nt) {
            xq[i] = ld(qb + (size_t)t0 * dqk + i);
            xk[i] = ld(kb + (size_t)t0 * dqk + i);
        }
        for (int i = tid; i < Lc * dv; i += nt) vs[i] = ld(vb + (size_t)t0 * dv + i);
        if (logdecay && warp == 0) {
            // the chunk's gates (C <= 32: one warp).  Every decay factor is a
            // plain sum of gates, never a difference of prefix sums, so a gate
            // of -inf gives exact zeros and large gates lose no precision.
            const float gj = lane < Lc ? logdecay[row0 + t0 + lane] : 0.f;
            float x = gj;   // inclusive prefix
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            float r = __shfl_down_sync(0xffffffffu, gj, 1);   // exclusive suffix over lanes j+1 .. Lc-1
            if (lane + 1 >= Lc) r = 0.f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, r, off);
                if (lane + off < 32) r += y;
            }
            if (lane < Lc) {
                cum[lane] = x;
                wk[lane] = expf(r);
                graw[lane] = gj;
            }
        }
        __syncthreads();
        for (int idx = tid; idx < Lc * F; idx += nt) {
            const int i = idx / F, f = idx - i * F;
            pq[i * FS + f] = phi_feature(fp, xq + i * dqk, f);
            pk[i * FS + f] = phi_feature(fp, xk + i * dqk, f);
        }
        __syncthreads();
        // Intra-chunk masked weights A_ij, j <= i (gated: times exp(L_i - L_j)).
        for (int idx = tid; idx < Lc * Lc; idx += nt) {
            const int i = idx / Lc, j = idx - i * Lc;
            float a = 0.f;
            if (j <= i) {
                for (int f = 0; f < F; ++f) a = fmaf(pq[i * FS + f], pk[j * FS + f], a);
                if (logdecay) {
                    float gsum = 0.f;   // g_{j+1} + ... + g_i
                    for (int l = j + 1; l <= i; ++l) gsum += graw[l];
                    a *= expf(gsum);
                }
            }
            A[i * C + j] = a;
        }
        __syncthreads();
        // den_i = sum_{j<=i} A_ij + e_i phi(q_i).z, e_i = exp(L_i) (1 ungated)  (one warp per row)
        for (int i = warp; i < Lc; i += nwarps) {
            float acc = 0.f;
            for (int f = lane; f < F; f += 32) acc = fmaf(pq[i * FS + f], z[f], acc);
            if (logdecay) acc *= expf(cum[i]);
            for (int j = lane; j <= i; j += 32) acc += A[i * C + j];
            for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) {
                den[i] = acc;
                if (den_out) den_out[row0 + t0 + i] = acc;
            }
        }
        __syncthreads();
        // num_i = sum_{j<=i} A_ij v_j + e_i phi(q_i) S ; y_i = num_i / den_i
        for (int idx = tid; idx < Lc * dv; idx += nt) {
            const int i = idx / dv, c = idx - i * dv;
            float acc = 0.f;
            for (int f = 0; f < F; ++f) acc = fmaf(pq[i * FS + f], S[f * DS + c], acc);
            if (logdecay) acc *= expf(cum[i]);
            for (int j = 0; j <= i; ++j) acc = fmaf(A[i * C + j], vs[j * dv + c], acc);
            st(ob + (size_t)(t0 + i) * dv + c, acc / den[i]);
        }
        __syncthreads();
        // S = e_last S + sum_j w_j phi(k_j) v_j^T ; z likewise (ungated: e = w = 1)
        const float e_last = logdecay ? expf(cum[Lc - 1]) : 1.f;
        for (int idx = tid; idx < F * dv; idx += nt) {
            const int f = idx / dv, c = idx - f * dv;
            float acc = S[f * DS + c] * e_last;
            if (logdecay)
                for (int j = 0; j < Lc; ++j) acc = fmaf(pk[j * FS + f] * wk[j], vs[j * dv + c], acc);
            else
                for (int j = 0; j < Lc; ++j) acc = fmaf(pk[j * FS + f], vs[j * dv + c], acc);
            S[f * DS + c] = acc;
        }
        for (int f = tid; f < F; f += nt) {
            float acc = z[f] * e_last;
            if (logdecay)
                for (int j = 0; j < Lc; ++j) acc = fmaf(pk[j * FS + f], wk[j], acc);
            else
                for (int j = 0; j < Lc; ++j) acc += pk[j * FS + f];
            z[f] = acc;
        }
    }
    __syncthreads();
    if (s_out)
        for (int idx = tid; idx < F * dv; idx += nt) {
            const int f = idx / dv, c = idx - f * dv;
            s_out[bh * F * dv + idx] = S[f * DS + c];
        }
    if (z_out)
        for (int f = tid; f < F; f += nt) z_out[bh * F + f] = z[f];
}

// ------------------------------------------------------------------ backward

struct SimtBwdSmem {
    int C, FS, DS;
    size_t floats(int F, int dqk, int dv) const
    {
        return (size_t)F * DS + F + 2 * (size_t)C * dqk + 3 * (size_t)C * FS +
               2 * (size_t)C * dv + 3 * (size_t)C * C + 6 * (size_t)C;
    }
};

inline SimtBwdSmem simt_bwd_layout(int C, int F, int dv)
{
    return SimtBwdSmem{C, odd_stride(F), odd_stride(dv)};
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
bwd_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                const T *__restrict__ dout, float *__restrict__ ws, T *__restrict__ dq,
                T *__restrict__ dk, T *__restrict__ dvo, int N, int dv, FmapParams fp, SimtBwdSmem L,
                const float *__restrict__ logdecay = nullptr, float *__restrict__ dlogdecay = nullptr)
{
    extern __shared__ float sm[];
    const int F = fp.F, dqk = fp.dqk, C = L.C, FS = L.FS, DS = L.DS;
    float *St = sm;                     // [F][DS]  S (pass 1) / R (pass 2)
    float *zt = St + (size_t)F * DS;    // [F]      z (pass 1) / r (pass 2)
    float *xq = zt + F;                 // [C][dqk]
    float *xk = xq + C * dqk;           // [C][dqk]
    float *pq = xk + C * dqk;           // [C][FS]
    float *pk = pq + (size_t)C * FS;    // [C][FS]
    float *dphi = pk + (size_t)C * FS;  // [C][FS]
    float *vs = dphi + (size_t)C * FS;  // [C][dv]
    float *gs = vs + C * dv;            // [C][dv]   dout_i, then g_i = dout_i / den_i
    float *A = gs + C * dv;             // [C][C]    a_ij
    float *dA = A + C * C;              // [C][C]    da_ij
    float *dd = dA + C * C;             // [C]       dden_i = -g_i . y_i
    float *dn = dd + C;                 // [C]       den_i
    // gated form (logdecay != null): w_ij = D_ij a_ij with D_ij = exp(g_{j+1} + ... + g_i)
    float *Dm = dn + C;                 // [C][C]    D_ij, j <= i
    float *cum = Dm + C * C;            // [C]       e_i: exp(g_{t0} + ... + g_{t0+i})
    float *wk = cum + C;                // [C]       f_j: exp(g_{t0+j+1} + ... + g_{last})
    float *graw = wk + C;               // [C]       the chunk's gates
    float *ub = graw + C;               // [C]       u_j = phi(k_j) . dphi(k_j)  (pass 2)
    double ucarry = 0.0;                // sum of u_j over the later chunks (pass 2); double:
                                        // the full sum is zero, so the partial sums cancel
    float elast = 1.f;                  // exp of the chunk's gate sum

    const int tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nwarps = nt >> 5;
    const size_t bh = blockIdx.x;
    const T *qb = q + bh * N * dqk, *kb = k + bh * N * dqk;
    const T *vb = v + bh * N * dv, *gb = dout + bh * N * dv;
    float *wsb = ws + bh * (size_t)N * 2;   // per token: den_i, dden_i (pass 1 -> pass 2)
    T *dqb = dq + bh * N * dqk, *dkb = dk + bh * N * dqk, *dvb = dvo + bh * N * dv;

    const int nchunks = (N + C - 1) / C;
    for (int pass = 0; pass < 2; ++pass) {
        __syncthreads();
        for (int i = tid; i < F * DS; i += nt) St[i] = 0.f;
        for (int i = tid; i < F; i += nt) zt[i] = 0.f;
        for (int cc = 0; cc < nchunks; ++cc) {
            const int chunk = pass == 0 ? cc : nchunks - 1 - cc;
            const int t0 = chunk * C;
            const int Lc = min(C, N - t0);
            __syncthreads();
            for (int i = tid; i < Lc * dqk; i += nt) {
                xq[i] = ld(qb + (size_t)t0 * dqk + i);
                xk[i] = ld(kb + (size_t)t0 * dqk + i);
            }
            for (int i = tid; i < Lc * dv; i += nt) {
                vs[i] = ld(vb + (size_t)t0 * dv + i);
                gs[i] = ld(gb + (size_t)t0 * dv + i);
            }
            if (logdecay && warp == 0) {
                // gate factors as plain sums of gates (as in the gated forward)
                const float gj = lane < Lc ? logdecay[bh * N + t0 + lane] : 0.f;
                float x = gj;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, off);
                    if (lane >= off) x += y;
                }
                float r = __shfl_down_sync(0xffffffffu, gj, 1);
                if (lane + 1 >= Lc) r = 0.f;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_down_sync(0xffffffffu, r, off);
                    if (lane + off < 32) r += y;
                }
                if (lane < Lc) {
                    cum[lane] = expf(x);
                    wk[lane] = expf(r);
                    graw[lane] = gj;
                }
            }
            __syncthreads();
            if (logdecay) {
                for (int idx = tid; idx < Lc * Lc; idx += nt) {
                    const int i = idx / Lc, j = idx - i * Lc;
                    float gsum = 0.f;
                    for (int l = j + 1; l <= i; ++l) gsum += graw[l];
                    Dm[i * C + j] = j <= i ? expf(gsum) : 0.f;
                }
                elast = cum[Lc - 1];
            }
            for (int idx = tid; idx < Lc * F; idx += nt) {
                const int i = idx / F, f = idx - i * F;
                pq[i * FS + f] = phi_feature(fp, xq + i * dqk, f);
                pk[i * FS + f] = phi_feature(fp, xk + i * dqk, f);
            }
            __syncthreads();
            // a_ij = phi(q_i).phi(k_j), j <= i (gated: w_ij = D_ij a_ij)
            for (int idx = tid; idx < Lc * Lc; idx += nt) {
                const int i = idx / Lc, j = idx - i * Lc;
                float a = 0.f;
                if (j <= i) {
                    for (int f = 0; f < F; ++f) a = fmaf(pq[i * FS + f], pk[j * FS + f], a);
                    if (logdecay) a *= Dm[i * C + j];
                }
                A[i * C + j] = a;
            }
            __syncthreads();
            if (pass == 0) {
                // den_i and y_i in fp32 from the state entering the chunk;
                // dden_i = -(dout_i . num_i) / den_i^2.  One warp per row.
                for (int i = warp; i < Lc; i += nwarps) {
                    const float ei = logdecay ? cum[i] : 1.f;
                    float d = 0.f;
                    for (int f = lane; f < F; f += 32) d = fmaf(pq[i * FS + f], zt[f], d);
                    d *= ei;
                    for (int j = lane; j <= i; j += 32) d += A[i * C + j];
                    for (int off = 16; off; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
                    float gy = 0.f;
                    for (int c = lane; c < dv; c += 32) {
                        float num = 0.f;
                        for (int f = 0; f < F; ++f) num = fmaf(pq[i * FS + f], St[f * DS + c], num);
                        num *= ei;
                        for (int j = 0; j <= i; ++j) num = fmaf(A[i * C + j], vs[j * dv + c], num);
                        gy = fmaf(gs[i * dv + c], num, gy);
                    }
                    for (int off = 16; off; off >>= 1) gy += __shfl_xor_sync(0xffffffffu, gy, off);
                    if (lane == 0) {
                        dn[i] = d;
                        dd[i] = -gy / (d * d);
                        wsb[2 * (t0 + i)] = d;
                        wsb[2 * (t0 + i) + 1] = dd[i];
                    }
                }
            } else {
                for (int i = tid; i < Lc; i += nt) {
                    dn[i] = wsb[2 * (t0 + i)];
                    dd[i] = wsb[2 * (t0 + i) + 1];
                }
            }
            __syncthreads();
            for (int i = tid; i < Lc * dv; i += nt) gs[i] = gs[i] / dn[i / dv];
            __syncthreads();
            // da_ij = g_i . v_j + dden_i for j <= i
            for (int idx = tid; idx < Lc * Lc; idx += nt) {
                const int i = idx / Lc, j = idx - i * Lc;
                float da = 0.f;
                if (j <= i) {
                    for (int c = 0; c < dv; ++c) da = fmaf(gs[i * dv + c], vs[j * dv + c], da);
                    da += dd[i];
                    if (logdecay) da *= Dm[i * C + j];   // dL/da_ij = D_ij dL/dw_ij
                }
                dA[i * C + j] = da;
            }
            __syncthreads();
            if (pass == 0) {
                // dphi(q_i) = sum_{j<=i, chunk} da_ij phi(k_j) + S g_i + z dden_i
                for (int idx = tid; idx < Lc * F; idx += nt) {
                    const int i = idx / F, f = idx - i * F;
                    float acc = zt[f] * dd[i];
                    for (int c = 0; c < dv; ++c) acc = fmaf(St[f * DS + c], gs[i * dv + c], acc);
                    if (logdecay) acc *= cum[i];
                    for (int j = 0; j <= i; ++j) acc = fmaf(dA[i * C + j], pk[j * FS + f], acc);
                    dphi[i * FS + f] = acc;
                }
                __syncthreads();
                for (int idx = tid; idx < Lc * dqk; idx += nt) {
                    const int i = idx / dqk, a = idx - i * dqk;
                    st(dqb + (size_t)t0 * dqk + idx, phi_vjp_component(fp, xq + i * dqk, dphi + i * FS, a));
                }
                // S = e_last S + sum_j f_j phi(k_j) v_j^T ; z likewise (ungated: factors 1)
                for (int idx = tid; idx < F * dv; idx += nt) {
                    const int f = idx / dv, c = idx - f * dv;
                    float acc = St[f * DS + c] * elast;
                    for (int j = 0; j < Lc; ++j)
                        acc = fmaf(logdecay ? pk[j * FS + f] * wk[j] : pk[j * FS + f], vs[j * dv + c], acc);
                    St[f * DS + c] = acc;
                }
                for (int f = tid; f < F; f += nt) {
                    float acc = zt[f] * elast;
                    for (int j = 0; j < Lc; ++j) acc += logdecay ? pk[j * FS + f] * wk[j] : pk[j * FS + f];
                    zt[f] = acc;
                }
            } else {
                // dphi(k_j) = sum_{i>=j, chunk} da_ij phi(q_i) + R v_j + r
                for (int idx = tid; idx < Lc * F; idx += nt) {
                    const int j = idx / F, f = idx - j * F;
                    float acc = zt[f];
                    for (int c = 0; c < dv; ++c) acc = fmaf(St[f * DS + c], vs[j * dv + c], acc);
                    if (logdecay) acc *= wk[j];
                    for (int i = j; i < Lc; ++i) acc = fmaf(dA[i * C + j], pq[i * FS + f], acc);
                    dphi[j * FS + f] = acc;
                }
                // dv_j = sum_{i>=j, chunk} a_ij g_i + R^T phi(k_j)   (gated: w_ij, f_j R)
                for (int idx = tid; idx < Lc * dv; idx += nt) {
                    const int j = idx / dv, c = idx - j * dv;
                    float acc = 0.f;
                    for (int f = 0; f < F; ++f) acc = fmaf(St[f * DS + c], pk[j * FS + f], acc);
                    if (logdecay) acc *= wk[j];
                    for (int i = j; i < Lc; ++i) acc = fmaf(A[i * C + j], gs[i * dv + c], acc);
                    st(dvb + (size_t)t0 * dv + idx, acc);
                }
                __syncthreads();
                if (logdecay) {
                    // dL/dg_l = -sum_{j>=l} phi(k_j) . dphi(k_j): the weights of each
                    // output row sum to one, so only the pairs crossing l remain
                    for (int j = warp; j < Lc; j += nwarps) {
                        float u = 0.f;
                        for (int f = lane; f < F; f += 32) u = fmaf(pk[j * FS + f], dphi[j * FS + f], u);
#pragma unroll
                        for (int off = 16; off; off >>= 1) u += __shfl_xor_sync(0xffffffffu, u, off);
                        if (lane == 0) ub[j] = u;
                    }
                    __syncthreads();
                    if (tid == 0) {
                        double acc = ucarry;
                        for (int j = Lc - 1; j >= 0; --j) {
                            acc += (double)ub[j];
                            dlogdecay[bh * N + t0 + j] = (float)-acc;
                        }
                        ucarry = acc;   // only thread 0 carries the running sum
                    }
                }
                for (int idx = tid; idx < Lc * dqk; idx += nt) {
                    const int j = idx / dqk, a = idx - j * dqk;
                    st(dkb + (size_t)t0 * dqk + idx, phi_vjp_component(fp, xk + j * dqk, dphi + j * FS, a));
                }
                // R = e_last R + sum_i e_i phi(q_i) g_i^T ; r likewise with dden_i (ungated: factors 1)
                for (int idx = tid; idx < F * dv; idx += nt) {
                    const int f = idx / dv, c = idx - f * dv;
                    float acc = St[f * DS + c] * elast;
                    for (int i = 0; i < Lc; ++i)
                        acc = fmaf(logdecay ? pq[i * FS + f] * cum[i] : pq[i * FS + f], gs[i * dv + c], acc);
                    St[f * DS + c] = acc;
                }
                for (int f = tid; f < F; f += nt) {
                    float acc = zt[f] * elast;
                    for (int i = 0; i < Lc; ++i)
                        acc = fmaf(logdecay ? pq[i * FS + f] * cum[i] : pq[i * FS + f], dd[i], acc);
                    zt[f] = acc;
                }
            }
        }
    }
}

// -------------------------------------------------------------------- decode

// One block per head; blockDim = dv * R threads, thread (r, c) owns column c
// of the state rows f = r, r + R, ...
template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
decode_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                   T *__restrict__ y, float *__restrict__ S, float *__restrict__ z, int dv,
                   FmapParams fp, const float *__restrict__ logdecay)
{
    extern __shared__ float sm[];
    const int F = fp.F, dqk = fp.dqk;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int R = nt / dv;
    float *pq = sm;            // [F]
    float *pk = pq + F;        // [F]
    float *xq = pk + F;        // [dqk]
    float *xk = xq + dqk;      // [dqk]
    float *vv = xk + dqk;      // [dv]
    float *red = vv + dv;      // [R][dv]
    float *wred = red + R * dv;  // [32]
    const size_t bh = blockIdx.x;

    for (int i = tid; i < dqk; i += nt) {
        xq[i] = ld(q + bh * dqk + i);
        xk[i] = ld(k + bh * dqk + i);
    }
    for (int i = tid; i < dv; i += nt) vv[i] = ld(v + bh * dv + i);
    __syncthreads();
    for (int f = tid; f < F; f += nt) {
        pq[f] = phi_feature(fp, xq, f);
        pk[f] = phi_feature(fp, xk, f);
    }
    __syncthreads();
    float *Sb = S + bh * F * dv;
    float *zb = z + bh * F;
    const float gate = logdecay ? expf(logdecay[bh]) : 1.f;   // forget gate (1 ungated)
    if (tid < R * dv) {
        const int r = tid / dv, c = tid - r * dv;
        const float vc = vv[c];
        float acc = 0.f;
        for (int f = r; f < F; f += R) {
            const float s = fmaf(pk[f], vc, gate * Sb[(size_t)f * dv + c]);
            Sb[(size_t)f * dv + c] = s;
            acc = fmaf(pq[f], s, acc);
        }
        red[r * dv + c] = acc;
    }
    float dacc = 0.f;
    for (int f = tid; f < F; f += nt) {
        const float zz = fmaf(gate, zb[f], pk[f]);
        zb[f] = zz;
        dacc = fmaf(pq[f], zz, dacc);
    }
    for (int off = 16; off; off >>= 1) dacc += __shfl_xor_sync(0xffffffffu, dacc, off);
    if ((tid & 31) == 0) wred[tid >> 5] = dacc;
    __syncthreads();
    if (tid < dv) {
        float den = 0.f;
        for (int w = 0; w < (nt + 31) / 32; ++w) den += wred[w];
        float num = 0.f;
        for (int r = 0; r < R; ++r) num += red[r * dv + tid];
        st(y + bh * dv + tid, num / den);
    }
}

// --------------------------------------------------------------- feature map

template <typename T>
__global__ void feature_map_kernel(const T *__restrict__ x, T *__restrict__ phi, int64_t rows,
                                   FmapParams fp)
{
    const int64_t total = rows * fp.F;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = idx / fp.F;
        const int f = (int)(idx - r * fp.F);
        // Only the coordinates this feature reads are loaded.
        const T *xr = x + r * fp.dqk;
        float val;
        if (fp.fmap == LA_FMAP_ELU1) {
            val = elu1(ld(xr + f));
        } else if (f == 0) {
            val = 1.f;
        } else if (f <= fp.dqk) {
            val = ld(xr + f - 1) * fp.inv_c1;
        } else if (fp.fmap == LA_FMAP_TAYLOR2_SYM) {
            const int i2 = f - 1 - fp.dqk;
            if (i2 < fp.dqk) {
                const float xa = ld(xr + i2);
                val = xa * xa * fp.inv_c2;
            } else {
                int a, b;
                sym_pair(i2 - fp.dqk, fp.dqk, a, b);
                val = ld(xr + a) * ld(xr + b) * fp.inv_c3;
            }
        } else {
            const int i2 = f - 1 - fp.dqk;
            const int a = i2 / fp.dqk, b = i2 - a * fp.dqk;
            val = ld(xr + a) * ld(xr + b) * fp.inv_c2;
        }
        st(phi + idx, val);
    }
}

}  // namespace la
