// la_fwd_ws_sm100.cuh -- warp-specialised chunked forward for the elu(x)+1
// map with d_qk = d_v = 64 (bf16 I/O), on tcgen05 tensor cores with TMA.
//
// Same mathematics as la_prefill_sm100.cuh (BASED page, Knowl 3 parallel
// form computed chunk by chunk as Knowl 5 describes: a masked quadratic term
// inside each 128-token chunk plus the product with the state of the earlier
// chunks), but the chunk's steps run on different warps so that consecutive
// chunks overlap.  Roles (512 threads):
//
//   warp 0        TMA producer: Q_c, K_c (SW128) and V_c (SW32 16-column
//                 blocks) into a 2-stage ring; ragged tails zero-filled.
//   warp 1        MMA issuer (one thread):
//                   X(c)  MMA1  A[c%2]  = phi(Q_c) phi(K_c)^T
//                         MMA3  dS      = phi(K_c)^T V_aug,c   (this chunk's increment)
//                   Y(c)  MMA2  O[c%2]  = P_c V_aug,c + phi(Q_c) S_snap(c)
//                 issued in the order X(c+1), Y(c) so the next chunk's scores
//                 run while this chunk's mask is being applied.
//   warps 4-7     phi: elu(x)+1 in place on the Q and K tiles (packed bf16x2
//                 exp2); key rows past N are zeroed so they add nothing.
//   warps 8-11    mask: A -> P = bf16(A masked to j <= i).
//   warps 12-15   state + output: S += dS in fp32 registers (feature rows in
//                 TMEM lanes), S_snap(c+1) = bf16(S) for the next MMA2, then
//                 y = O[:, :64] / O[:, 64] to global memory.
//
// V_aug = [V | 1 | 0 ...] (80 columns), so S_aug = [S | z] and O = [num | den]
// come out of the same MMAs.  Only dS(c) -> S_snap(c+1) -> MMA2(c+1) is
// serial across chunks.  Every wait is bounded (2 s); on expiry the kernel
// records a timeout in the status word, stops issuing, frees TMEM and exits.
//
// MODE 1 computes, for each segment but the last, the increment of the
// segment's state into the workspace (TMA K/V, phi of K, MMA3 accumulated
// over the segment's chunks); MODE 0 starts each segment from the sum of the
// increments of the segments before it.
#pragma once

#include "la_device.cuh"
#include "la_prefill_sm100.cuh"
#include "sm100.cuh"

namespace la {

struct WsCfg64 {
    static constexpr int C = 128, DQK = 64, DV = 64, NA = 80;
    static constexpr int NS = 2;                         // TMA stages
    static constexpr int QK_TILE = C * DQK * 2;          // 16 KB
    static constexpr int V_BLK = C * 32;                 // 4 KB (16 columns)
    static constexpr int V_TILE = (DV / 16 + 1) * V_BLK; // 20 KB incl. the ones block
    static constexpr int STAGE = 2 * QK_TILE + V_TILE;   // 52 KB
    static constexpr int P_TILE = C * C * 2;             // 32 KB
    static constexpr int S_BLK = DQK * 32;               // 2 KB (16 columns x 64 feature rows)
    static constexpr int S_TILE = (NA / 16) * S_BLK;     // 10 KB
    static constexpr int OFF_STAGE = 0;
    static constexpr int OFF_P = OFF_STAGE + NS * STAGE;         // 104 KB
    static constexpr int OFF_S = OFF_P + 2 * P_TILE;             // 168 KB
    static constexpr int OFF_BAR = OFF_S + 2 * S_TILE;           // 188 KB
    static constexpr int SMEM_ALLOC = OFF_BAR + 256 + 1024;
    // TMEM columns
    static constexpr int COL_A = 0;      // 2 x 128
    static constexpr int COL_O = 256;    // 2 x 80
    static constexpr int COL_DS = 416;   // 80 (M = 64 layout: feature f in lane 32*(f/16) + f%16)
    static constexpr int TMEM_COLS = 512;
    static constexpr int TX_BYTES = 2 * QK_TILE + DV * C * 2;
};

namespace ws_detail {

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(sm100::smem_addr(bar)) : "memory");
}

// elu(x)+1 on two packed bf16 values: max(x,0) + 2^(min(x,0) log2 e).  The
// exponent argument is formed in fp32 and rounded once to bf16; the packed
// exp2 returns bf16, the precision the MMA consumes.
__device__ __forceinline__ uint32_t elu1_bf16x2(uint32_t x)
{
    const uint32_t zero = 0u;
    uint32_t neg, pos;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(neg) : "r"(x), "r"(zero));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(pos) : "r"(x), "r"(zero));
    const float lo = __uint_as_float(neg << 16) * 1.4426950408889634f;
    const float hi = __uint_as_float(neg & 0xFFFF0000u) * 1.4426950408889634f;
    uint32_t arg, ex, r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(arg) : "f"(hi), "f"(lo));
    asm("ex2.approx.ftz.bf16x2 %0, %1;" : "=r"(ex) : "r"(arg));
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(pos), "r"(ex));
    return r;
}

__device__ __forceinline__ uint4 lds128(uint32_t a)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
    return r;
}

__device__ __forceinline__ void sts128(uint32_t a, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

}  // namespace ws_detail

template <int MODE>
__global__ void __launch_bounds__(512, 1)
fwd_ws_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const FwdParams p)
{
    using namespace sm100;
    using namespace fwd_detail;
    using namespace ws_detail;
    using Cfg = WsCfg64;
    constexpr int C = Cfg::C, NA = Cfg::NA, DV = Cfg::DV, NS = Cfg::NS, FP = Cfg::DQK;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *full = bars + 0;       // [NS] TMA landed
    uint64_t *empty = bars + 2;      // [NS] stage released by the last MMA reading it
    uint64_t *phi_done = bars + 4;   // [NS] phi written (4 warp arrivals)
    uint64_t *a_full = bars + 6;     // [2] MMA1 done
    uint64_t *p_full = bars + 8;     // [2] P written, A read (4)
    uint64_t *o_full = bars + 10;    // [2] MMA2 done
    uint64_t *o_free = bars + 12;    // [2] O read (4)
    uint64_t *snap_full = bars + 14; // [2] S_snap written (4)
    uint64_t *ds_full = bars + 16;   // MMA3 done
    uint64_t *ds_free = bars + 17;   // dS read (4)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 18);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 19);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x / p.P, seg = blockIdx.x % p.P;
    if (MODE == 1 && seg == p.P - 1) return;
    const int c_begin = seg * p.cps;
    const int c_end = min(p.nchunks, c_begin + p.cps);
    const int nit = c_end - c_begin;
    const int N = p.N;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&phi_done[s], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&a_full[b], 1);
            mbar_init(&p_full[b], 4);
            mbar_init(&o_full[b], 1);
            mbar_init(&o_free[b], 4);
            mbar_init(&snap_full[b], 4);
        }
        mbar_init(ds_full, 1);
        mbar_init(ds_free, 4);
        *abort_flag = 0;
        mbar_init_fence();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 0) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    // Normaliser block of each stage's V_aug: column 0 = 1 (overall column 64).
    if (tid < 128)
        for (int s = 0; s < NS; ++s) {
            uint8_t *blk = smem + Cfg::OFF_STAGE + s * Cfg::STAGE + 2 * Cfg::QK_TILE + (DV / 16) * Cfg::V_BLK;
            const int r = tid;
            uint4 *row = reinterpret_cast<uint4 *>(blk + (r >> 3) * 256 + (r & 7) * 32);
            const int one_chunk = (r >> 2) & 1;
            row[one_chunk] = make_uint4(pack_bf16(1.f, 0.f), 0u, 0u, 0u);
            row[one_chunk ^ 1] = make_uint4(0u, 0u, 0u, 0u);
        }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto stage_ptr = [&](int s) { return smem + Cfg::OFF_STAGE + s * Cfg::STAGE; };
    auto fail = [&]() { *abort_flag = 1; };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            for (int it = 0; it < nit && !*abort_flag; ++it) {
                const int s = it % NS;
                if (it >= NS && !mbar_wait(&empty[s], ((it / NS) - 1) & 1)) { fail(); break; }
                const int t0 = (c_begin + it) * C;
                uint8_t *st = stage_ptr(s);
                mbar_arrive_expect_tx(&full[s], MODE == 0 ? Cfg::TX_BYTES : Cfg::TX_BYTES - Cfg::QK_TILE);
                if (MODE == 0) tma_load_3d(st, &tm_q, &full[s], 0, t0, bh);
                tma_load_3d(st + Cfg::QK_TILE, &tm_k, &full[s], 0, t0, bh);
                for (int x = 0; x < DV; x += 16)
                    tma_load_3d(st + 2 * Cfg::QK_TILE + (x / 16) * Cfg::V_BLK, &tm_v, &full[s], x, t0, bh);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
            const uint32_t id_s = idesc_bf16(64, NA, 1, 1);
            const uint32_t id_o = idesc_bf16(128, NA, 0, 1);
            // X(it): scores and state increment of chunk it
            auto issue_x = [&](int it) -> bool {
                const int s = it % NS;
                if (!mbar_wait(&full[s], (it / NS) & 1)) return false;
                if (!mbar_wait(&phi_done[s], (it / NS) & 1)) return false;
                tc_fence_after();
                const uint32_t aQ = smem_addr(stage_ptr(s)), aK = aQ + Cfg::QK_TILE, aV = aK + Cfg::QK_TILE;
                if (MODE == 0) {
                    const uint32_t dA = tmem + Cfg::COL_A + (it & 1) * 128;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(dA, smem_desc(aQ + kk * 32, 16, 1024, kSw128), smem_desc(aK + kk * 32, 16, 1024, kSw128),
                                 id_qk, kk > 0);
                    mma_commit(&a_full[it & 1]);
                    if (it >= 1) {
                        if (!mbar_wait(ds_free, (it - 1) & 1)) return false;
                        tc_fence_after();
                    }
                }
                const bool acc_prev = (MODE == 1) && it > 0;  // MODE 1 sums the whole segment
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + Cfg::COL_DS, smem_desc(aK + kk * 2048, C * 128, 1024, kSw128),
                             smem_desc(aV + kk * 512, Cfg::V_BLK, 256, kSw32), id_s, acc_prev || kk > 0);
                if (MODE == 0) mma_commit(ds_full);
                else mma_commit(&empty[s]);
                return true;
            };
            // Y(it): output of chunk it
            auto issue_y = [&](int it) -> bool {
                const int s = it % NS, b = it & 1;
                if (!mbar_wait(&p_full[b], (it >> 1) & 1)) return false;
                if (!mbar_wait(&snap_full[it & 1], (it >> 1) & 1)) return false;   // snapshot index it
                if (it >= 2 && !mbar_wait(&o_free[b], ((it >> 1) - 1) & 1)) return false;
                tc_fence_after();
                const uint32_t aQ = smem_addr(stage_ptr(s)), aV = aQ + 2 * Cfg::QK_TILE;
                const uint32_t aP = smem_addr(smem + Cfg::OFF_P + b * Cfg::P_TILE);
                const uint32_t aS = smem_addr(smem + Cfg::OFF_S + (it & 1) * Cfg::S_TILE);
                const uint32_t dO = tmem + Cfg::COL_O + b * NA;
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(dO, smem_desc(aP + (kk >> 2) * (C * 128) + (kk & 3) * 32, 16, 1024, kSw128),
                             smem_desc(aV + kk * 512, Cfg::V_BLK, 256, kSw32), id_o, kk > 0);
#pragma unroll
                for (int kk = 0; kk < FP / 16; ++kk)
                    mma_bf16(dO, smem_desc(aQ + kk * 32, 16, 1024, kSw128),
                             smem_desc(aS + kk * 512, Cfg::S_BLK, 256, kSw32), id_o, true);
                mma_commit(&o_full[b]);
                mma_commit(&empty[s]);
                return true;
            };
            bool ok = nit > 0 ? issue_x(0) : true;
            for (int it = 0; it < nit && ok && !*abort_flag; ++it) {
                if (it + 1 < nit) ok = issue_x(it + 1);
                if (ok && MODE == 0) ok = issue_y(it);
            }
            if (ok && MODE == 1) mma_commit(ds_full);   // segment increment complete
            if (!ok) fail();
        }
    } else if (warp >= 4 && warp < 8) {
        // ---------------------------------------------------------------- phi
        const int i = tid - 128;
        for (int it = 0; it < nit && !*abort_flag; ++it) {
            const int s = it % NS;
            if (!mbar_wait(&full[s], (it / NS) & 1)) { fail(); break; }
            const int t0 = (c_begin + it) * C;
            const bool kvalid = t0 + i < N;
            const uint32_t base = smem_addr(stage_ptr(s));
#pragma unroll
            for (int m = (MODE == 0 ? 0 : 1); m < 2; ++m) {
                const uint32_t tile = base + m * Cfg::QK_TILE;
                const bool zero = (m == 1) && !kvalid;
                uint4 raw[8];
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) raw[cc] = lds128(tile + sw128_off(i, cc * 8));
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    uint4 r = raw[cc];
                    r = zero ? make_uint4(0u, 0u, 0u, 0u)
                             : make_uint4(elu1_bf16x2(r.x), elu1_bf16x2(r.y), elu1_bf16x2(r.z), elu1_bf16x2(r.w));
                    sts128(tile + sw128_off(i, cc * 8), r);
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&phi_done[s]);
        }
    } else if (warp >= 8 && warp < 12) {
        // --------------------------------------------------------------- mask
        if (MODE == 0) {
            const int i = tid - 256;
            const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
            for (int it = 0; it < nit && !*abort_flag; ++it) {
                const int b = it & 1;
                if (!mbar_wait(&a_full[b], (it >> 1) & 1)) { fail(); break; }
                // P[b] was last read by MMA2(it-2)
                if (it >= 2 && !mbar_wait(&o_full[b], ((it >> 1) - 1) & 1)) { fail(); break; }
                tc_fence_after();
                const uint32_t aP = smem_addr(smem + Cfg::OFF_P + b * Cfg::P_TILE);
                const uint32_t tA = tmem + lane_base + Cfg::COL_A + b * 128;
#pragma unroll 1
                for (int j0 = 0; j0 < C; j0 += 64) {
                    float a[64];
                    tmem_ld32(tA + j0, a);
                    tmem_ld32(tA + j0 + 32, a + 32);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 64; e += 8) {
                        float w[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) w[u] = (j0 + e + u <= i) ? a[e + u] : 0.f;
                        sts128(aP + sw128_off(i, j0 + e),
                               make_uint4(pack_bf16(w[0], w[1]), pack_bf16(w[2], w[3]), pack_bf16(w[4], w[5]),
                                          pack_bf16(w[6], w[7])));
                    }
                }
                fence_proxy_async();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[b]);
            }
        }
    } else if (warp >= 12) {
        // ------------------------------------------------- state and output
        const int wq = warp & 3;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const int f = wq * 16 + lane;            // feature row of dS held by this lane (lane < 16)
        const bool frow = lane < 16;
        float S[NA];
#pragma unroll
        for (int e = 0; e < NA; ++e) S[e] = 0.f;
        if (MODE == 0 && seg > 0 && frow) {
            for (int s2 = 0; s2 < seg; ++s2) {
                const float *src = p.ws + ((size_t)(bh * p.P + s2) * FP + f) * NA;
#pragma unroll
                for (int e = 0; e < NA; ++e) S[e] += src[e];
            }
        }
        auto write_snap = [&](int j) {   // snapshot j = state before chunk j, buffer j & 1
            if (frow) {
                const uint32_t aS = smem_addr(smem + Cfg::OFF_S + (j & 1) * Cfg::S_TILE);
#pragma unroll
                for (int c0 = 0; c0 < NA; c0 += 8)
                    sts128(aS + sw32_off(f, c0, FP),
                           make_uint4(pack_bf16(S[c0], S[c0 + 1]), pack_bf16(S[c0 + 2], S[c0 + 3]),
                                      pack_bf16(S[c0 + 4], S[c0 + 5]), pack_bf16(S[c0 + 6], S[c0 + 7])));
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&snap_full[j & 1]);
        };
        if (MODE == 0) {
            write_snap(0);
            for (int it = 0; it < nit && !*abort_flag; ++it) {
                // dS(it) -> S, snapshot it+1 (buffer last read by MMA2(it-1), already complete)
                if (!mbar_wait(ds_full, it & 1)) { fail(); break; }
                tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < NA; c0 += 16) {
                    float d[16];
                    tmem_ld16(tmem + lane_base + Cfg::COL_DS + c0, d);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) S[c0 + e] += d[e];
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(ds_free);
                if (it + 1 < nit) write_snap(it + 1);
                // output of chunk it
                const int b = it & 1;
                if (!mbar_wait(&o_full[b], (it >> 1) & 1)) { fail(); break; }
                tc_fence_after();
                const int t0 = (c_begin + it) * C;
                const int row = wq * 32 + lane;
                float den[16];
                tmem_ld16(tmem + lane_base + Cfg::COL_O + b * NA + DV, den);
                tmem_ld_wait();
                const float inv = 1.f / den[0];
                __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) + ((size_t)bh * N + t0 + row) * DV;
                const bool valid = t0 + row < N;
#pragma unroll
                for (int c0 = 0; c0 < DV; c0 += 16) {
                    float o[16];
                    tmem_ld16(tmem + lane_base + Cfg::COL_O + b * NA + c0, o);
                    tmem_ld_wait();
                    if (valid) {
                        *reinterpret_cast<uint4 *>(orow + c0) =
                            make_uint4(pack_bf16(o[0] * inv, o[1] * inv), pack_bf16(o[2] * inv, o[3] * inv),
                                       pack_bf16(o[4] * inv, o[5] * inv), pack_bf16(o[6] * inv, o[7] * inv));
                        *reinterpret_cast<uint4 *>(orow + c0 + 8) =
                            make_uint4(pack_bf16(o[8] * inv, o[9] * inv), pack_bf16(o[10] * inv, o[11] * inv),
                                       pack_bf16(o[12] * inv, o[13] * inv), pack_bf16(o[14] * inv, o[15] * inv));
                    }
                }
                if (valid && p.den_out) p.den_out[(size_t)bh * N + t0 + row] = den[0];
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&o_free[b]);
            }
            // final state of the sequence (last segment only)
            if (seg == p.P - 1 && frow && !*abort_flag) {
                if (p.s_out) {
                    float *dst = p.s_out + ((size_t)bh * FP + f) * DV;
#pragma unroll
                    for (int e = 0; e < DV; ++e) dst[e] = S[e];
                }
                if (p.z_out) p.z_out[(size_t)bh * FP + f] = S[DV];
            }
        } else {
            // MODE 1: the accumulated increment of this segment -> workspace
            if (nit > 0) {
                if (mbar_wait(ds_full, 0)) {
                    tc_fence_after();
                    float *dst = p.ws + ((size_t)(bh * p.P + seg) * FP + f) * NA;
#pragma unroll
                    for (int c0 = 0; c0 < NA; c0 += 16) {
                        float d[16];
                        tmem_ld16(tmem + lane_base + Cfg::COL_DS + c0, d);
                        tmem_ld_wait();
                        if (frow)
#pragma unroll
                            for (int e = 0; e < 16; ++e) dst[c0 + e] = d[e];
                    }
                } else {
                    fail();
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

}  // namespace la
