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

// Optional per-role timeline of block 0 (clock64 at role boundaries, per
// chunk), for profiling builds that define LA_TIMELINE; compiled out
// otherwise.
#ifdef LA_TIMELINE
__device__ long long g_timeline[2][16][64];
#define LA_TL(ev, it_)                                                         \
    do {                                                                       \
        if (blockIdx.x == 0 && (it_) >= 0 && (it_) < 64) g_timeline[MODE][ev][(it_)] = clock64(); \
    } while (0)
#else
#define LA_TL(ev, it_) do { } while (0)
#endif

template <int MODE>
struct WsCfg64 {
    static constexpr int C = 128, DQK = 64, DV = 64, NA = 80;
    // MODE 0 stages hold Q, K and V_aug; MODE 1 (state increments) only K and V_aug.
    static constexpr int NS = MODE == 0 ? 3 : 4;         // TMA stages
    static constexpr int QK_TILE = C * DQK * 2;          // 16 KB
    static constexpr int V_BLK = C * 32;                 // 4 KB (16 columns)
    static constexpr int V_TILE = (DV / 16 + 1) * V_BLK; // 20 KB incl. the ones block
    static constexpr int OFF_Q = 0;                      // within a stage (MODE 0 only)
    static constexpr int OFF_K = MODE == 0 ? QK_TILE : 0;
    static constexpr int OFF_V = OFF_K + QK_TILE;
    static constexpr int STAGE = OFF_V + V_TILE;         // 52 KB / 36 KB
    static constexpr int S_BLK = DQK * 32;               // 2 KB (16 columns x 64 feature rows)
    static constexpr int S_TILE = (NA / 16) * S_BLK;     // 10 KB
    static constexpr int OFF_STAGE = 0;
    static constexpr int OFF_S = OFF_STAGE + NS * STAGE;
    static constexpr int OFF_BAR = OFF_S + (MODE == 0 ? 2 * S_TILE : 0);
    static constexpr int SMEM_ALLOC = OFF_BAR + 256 + 1024;
    // TMEM columns
    static constexpr int COL_A = 0;      // 2 x 128 (scores fp32; then P bf16 packed in the first 64)
    static constexpr int COL_O = 256;    // 2 x 80
    static constexpr int COL_DS = 416;   // 80 (M = 64 layout: feature f in lane 32*(f/16) + f%16)
    static constexpr int TMEM_COLS = 512;
    static constexpr int TX_BYTES = (MODE == 0 ? 2 : 1) * QK_TILE + DV * C * 2;
    static constexpr int PREFETCH = 4;   // chunks ahead whose tiles are pulled into L2
};

namespace ws_detail {

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(sm100::smem_addr(bar)) : "memory");
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
    using Cfg = WsCfg64<MODE>;
    constexpr int C = Cfg::C, NA = Cfg::NA, DV = Cfg::DV, NS = Cfg::NS, FP = Cfg::DQK;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *full = bars + 0;       // [NS] TMA landed
    uint64_t *empty = bars + 4;      // [NS] stage released by the last MMA reading it
    uint64_t *phi_done = bars + 8;   // [NS] phi written (4 warp arrivals)
    uint64_t *a_full = bars + 12;    // [2] MMA1 done
    uint64_t *p_full = bars + 14;    // [2] P written, A read (4)
    uint64_t *o_full = bars + 16;    // [2] MMA2 done
    uint64_t *o_free = bars + 18;    // [2] O read (4)
    uint64_t *snap_full = bars + 20; // [2] S_snap written (4)
    uint64_t *ds_full = bars + 22;   // MMA3 done
    uint64_t *ds_free = bars + 23;   // dS read (4)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 24);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 25);

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
            mbar_init(&phi_done[s], MODE == 0 ? 6 : 4);
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
            uint8_t *blk = smem + Cfg::OFF_STAGE + s * Cfg::STAGE + Cfg::OFF_V + (DV / 16) * Cfg::V_BLK;
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
    if (tid == 0) LA_TL(13, 0);

    auto stage_ptr = [&](int s) { return smem + Cfg::OFF_STAGE + s * Cfg::STAGE; };
    auto fail = [&]() { *abort_flag = 1; };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            auto prefetch = [&](int it) {
                const int t0 = (c_begin + it) * C;
                if (MODE == 0) tma_prefetch_3d(&tm_q, 0, t0, bh);
                tma_prefetch_3d(&tm_k, 0, t0, bh);
                for (int x = 0; x < DV; x += 16) tma_prefetch_3d(&tm_v, x, t0, bh);
            };
            for (int it = 0; it < nit && !*abort_flag; ++it) {
                if (it == NS)
                    for (int j = NS; j < nit && j < NS + Cfg::PREFETCH; ++j) prefetch(j);
                const int s = it % NS;
                if (it >= NS && !mbar_wait(&empty[s], ((it / NS) - 1) & 1)) { fail(); break; }
                const int t0 = (c_begin + it) * C;
                uint8_t *st = stage_ptr(s);
                LA_TL(0, it);
                mbar_arrive_expect_tx(&full[s], Cfg::TX_BYTES);
                if (MODE == 0) tma_load_3d(st + Cfg::OFF_Q, &tm_q, &full[s], 0, t0, bh);
                tma_load_3d(st + Cfg::OFF_K, &tm_k, &full[s], 0, t0, bh);
                for (int x = 0; x < DV; x += 16)
                    tma_load_3d(st + Cfg::OFF_V + (x / 16) * Cfg::V_BLK, &tm_v, &full[s], x, t0, bh);
                if (it + NS + Cfg::PREFETCH < nit) prefetch(it + NS + Cfg::PREFETCH);
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
                LA_TL(1, it);
                tc_fence_after();
                const uint32_t st = smem_addr(stage_ptr(s));
                const uint32_t aQ = st + Cfg::OFF_Q, aK = st + Cfg::OFF_K, aV = st + Cfg::OFF_V;
                if (MODE == 0) {
                    const uint32_t dA = tmem + Cfg::COL_A + (it & 1) * 128;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(dA, smem_desc(aQ + kk * 32, 16, 1024, kSw128), smem_desc(aK + kk * 32, 16, 1024, kSw128),
                                 id_qk, kk > 0);
                    mma_commit(&a_full[it & 1]);
                    if (!mbar_wait(ds_free, it & 1)) return false;   // S(it-1) read / initial state stored
                    tc_fence_after();
                }
                // MODE 0 accumulates onto the state in TMEM; MODE 1 sums the segment from zero
                const bool acc_prev = (MODE == 0) || it > 0;
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + Cfg::COL_DS, smem_desc(aK + kk * 2048, C * 128, 1024, kSw128),
                             smem_desc(aV + kk * 512, Cfg::V_BLK, 256, kSw32), id_s, acc_prev || kk > 0);
                if (MODE == 0) mma_commit(ds_full);
                else mma_commit(&empty[s]);
                LA_TL(2, it);
                return true;
            };
            // Y(it): output of chunk it
            auto issue_y = [&](int it) -> bool {
                const int s = it % NS, b = it & 1;
                if (!mbar_wait(&p_full[b], (it >> 1) & 1)) return false;
                if (!mbar_wait(&snap_full[it & 1], (it >> 1) & 1)) return false;   // snapshot index it
                if (it >= 2 && !mbar_wait(&o_free[b], ((it >> 1) - 1) & 1)) return false;
                LA_TL(3, it);
                tc_fence_after();
                const uint32_t st = smem_addr(stage_ptr(s));
                const uint32_t aQ = st + Cfg::OFF_Q, aV = st + Cfg::OFF_V;
                const uint32_t tP = tmem + Cfg::COL_A + b * 128;   // P(it), bf16 pairs per column
                const uint32_t aS = smem_addr(smem + Cfg::OFF_S + (it & 1) * Cfg::S_TILE);
                const uint32_t dO = tmem + Cfg::COL_O + b * NA;
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16_ts(dO, tP + kk * 8, smem_desc(aV + kk * 512, Cfg::V_BLK, 256, kSw32), id_o, kk > 0);
#pragma unroll
                for (int kk = 0; kk < FP / 16; ++kk)
                    mma_bf16(dO, smem_desc(aQ + kk * 32, 16, 1024, kSw128),
                             smem_desc(aS + kk * 512, Cfg::S_BLK, 256, kSw32), id_o, true);
                mma_commit(&o_full[b]);
                mma_commit(&empty[s]);
                LA_TL(4, it);
                return true;
            };
            bool ok = true;
            if (MODE == 1) {
                for (int it = 0; it < nit && ok && !*abort_flag; ++it) ok = issue_x(it);
                if (ok) mma_commit(ds_full);   // segment increment complete
            } else {
                // Issue whichever of Y(ny) (output of the oldest pending chunk) and
                // X(nx) (scores and increment of the next chunk) has its inputs
                // ready, preferring Y; give up after 2 s without progress.
                auto x_ready = [&](int it) {
                    const int s = it % NS;
                    return mbar_test(&full[s], (it / NS) & 1) && mbar_test(&phi_done[s], (it / NS) & 1) &&
                           mbar_test(ds_free, it & 1);
                };
                auto y_ready = [&](int it) {
                    const int b = it & 1;
                    return mbar_test(&p_full[b], (it >> 1) & 1) && mbar_test(&snap_full[b], (it >> 1) & 1) &&
                           (it < 2 || mbar_test(&o_free[b], ((it >> 1) - 1) & 1));
                };
                int nx = 0, ny = 0;
                uint64_t t_last;
                asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_last));
                while (ny < nit && ok && !*abort_flag) {
                    bool progress = false;
                    if (ny < nx && y_ready(ny)) {
                        ok = issue_y(ny++);
                        progress = true;
                    } else if (nx < nit && nx <= ny + 1 && x_ready(nx)) {
                        ok = issue_x(nx++);
                        progress = true;
                    }
                    uint64_t t;
                    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
                    if (progress) {
                        t_last = t;
                    } else if (t - t_last > 2000000000ull) {
                        report(kStatusTimeout);
                        ok = false;
                    } else {
                        __nanosleep(64);   // leave issue slots to the warps sharing this SMSP
                    }
                }
            }
            if (!ok) fail();
        }
    } else if ((MODE == 0 && warp >= 2 && warp < 8) || (MODE == 1 && warp >= 4 && warp < 12)) {
        // ---------------------------------------------------------------- phi
        // elu(x)+1 in place.  MODE 0: warps 2-7 (192 threads) share the 512
        // half-rows (32 values) of the Q and K tiles of every chunk.  MODE 1:
        // only K; warps 4-7 take even chunks and warps 8-11 odd ones, a row
        // per thread.
        const int first = (MODE == 1 && warp >= 8) ? 1 : 0;
        const int step = MODE == 1 ? 2 : 1;
        const int pt = MODE == 0 ? tid - 64 : (tid & 127);   // 0..191 or 0..127
        for (int it = first; it < nit && !*abort_flag; it += step) {
            const int s = it % NS;
            if (!mbar_wait(&full[s], (it / NS) & 1)) { fail(); break; }
            if (pt == 0) LA_TL(5, it);
            const int t0 = (c_begin + it) * C;
            const uint32_t base = smem_addr(stage_ptr(s));
            auto half_row = [&](int m, int row, int h) {
                const uint32_t tile = base + (m == 0 ? Cfg::OFF_Q : Cfg::OFF_K);
                const bool zero = (m == 1) && (t0 + row >= N);
                uint4 raw[4];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) raw[cc] = lds128(tile + sw128_off(row, (h * 4 + cc) * 8));
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 r = raw[cc];
                    r = zero ? make_uint4(0u, 0u, 0u, 0u)
                             : make_uint4(elu1_bf16x2(r.x), elu1_bf16x2(r.y), elu1_bf16x2(r.z), elu1_bf16x2(r.w));
                    sts128(tile + sw128_off(row, (h * 4 + cc) * 8), r);
                }
            };
            if (MODE == 0) {
                for (int item = pt; item < 2 * C * 2; item += 192)   // item = (tile, row, half)
                    half_row(item >> 8, (item >> 1) & (C - 1), item & 1);
            } else {
                half_row(1, pt, 0);
                half_row(1, pt, 1);
            }
            fence_proxy_async();
            __syncwarp();
            if (pt == 0) LA_TL(6, it);
            if (lane == 0) mbar_arrive(&phi_done[s]);
        }
    } else if (warp >= 8 && warp < 12) {
        // --------------------------------------------------------------- mask
        {
            const int i = tid - 256;
            const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
            for (int it = 0; it < nit && !*abort_flag; ++it) {
                const int b = it & 1;
                if (!mbar_wait(&a_full[b], (it >> 1) & 1)) { fail(); break; }
                // P(it) overwrites the first 64 columns of A[b]: MMA2(it-2), the
                // last reader of the P in this buffer, finished before MMA1(it)
                // (MMAs execute in issue order).
                if (i == 0) LA_TL(7, it);
                tc_fence_after();
                const uint32_t tA = tmem + lane_base + Cfg::COL_A + b * 128;
#pragma unroll 1
                for (int j0 = 0; j0 < C; j0 += 64) {
                    float a[64];
                    tmem_ld32(tA + j0, a);
                    tmem_ld32(tA + j0 + 32, a + 32);
                    tmem_ld_wait();
                    uint32_t pk[32];
#pragma unroll
                    for (int e = 0; e < 64; e += 2)
                        pk[e / 2] = pack_bf16((j0 + e <= i) ? a[e] : 0.f, (j0 + e + 1 <= i) ? a[e + 1] : 0.f);
                    tmem_st32(tA + j0 / 2, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (i == 0) LA_TL(8, it);
                if (lane == 0) mbar_arrive(&p_full[b]);
            }
        }
    } else if (warp >= 12) {
        // ------------------------------------------------- state and output
        // The running state S_aug lives in TMEM (COL_DS, feature rows in the
        // lanes of the M = 64 layout); MMA3 accumulates each chunk into it.
        const int wq = warp & 3;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + lane_base + Cfg::COL_DS;
        const int f = wq * 16 + lane;            // feature row held by this lane (lane < 16)
        const bool frow = lane < 16;
        // snapshot j = state before chunk j (bf16, buffer j & 1) from 16-column batches
        auto snap_cols = [&](int j, int c0, const float *v) {
            if (frow) {
                const uint32_t aS = smem_addr(smem + Cfg::OFF_S + (j & 1) * Cfg::S_TILE);
                sts128(aS + sw32_off(f, c0, FP), make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                                            pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7])));
                sts128(aS + sw32_off(f, c0 + 8, FP),
                       make_uint4(pack_bf16(v[8], v[9]), pack_bf16(v[10], v[11]), pack_bf16(v[12], v[13]),
                                  pack_bf16(v[14], v[15])));
            }
        };
        auto snap_done = [&](int j) {
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&snap_full[j & 1]);
        };
        if (MODE == 0) {
            // initial state: the sum of the earlier segments' increments, or zero
            for (int c0 = 0; c0 < NA; c0 += 16) {
                float v[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = 0.f;
                if (seg > 0 && frow)
                    for (int s2 = 0; s2 < seg; ++s2) {
                        const float *src = p.ws + ((size_t)(bh * p.P + s2) * FP + f) * NA + c0;
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] += src[e];
                    }
                tmem_st16(tS + c0, v);
                snap_cols(0, c0, v);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ds_free);   // completion 0: initial state in TMEM
            snap_done(0);
            for (int it = 0; it < nit && !*abort_flag; ++it) {
                // state after chunk it -> snapshot it+1 (its buffer was last read by
                // MMA2(it-1), complete since the output of chunk it-1 was taken)
                if (!mbar_wait(ds_full, it & 1)) { fail(); break; }
                if (tid == 384) LA_TL(9, it);
                tc_fence_after();
                if (it + 1 < nit) {
#pragma unroll
                    for (int c0 = 0; c0 < NA; c0 += 48) {
                        float v[48];
                        tmem_ld16(tS + c0, v);
                        tmem_ld16(tS + c0 + 16, v + 16);
                        if (c0 + 32 < NA) tmem_ld16(tS + c0 + 32, v + 32);
                        tmem_ld_wait();
                        snap_cols(it + 1, c0, v);
                        snap_cols(it + 1, c0 + 16, v + 16);
                        if (c0 + 32 < NA) snap_cols(it + 1, c0 + 32, v + 32);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(ds_free);   // completion it+1: S(it) read
                if (it + 1 < nit) snap_done(it + 1);
                if (tid == 384) LA_TL(10, it);
                // output of chunk it
                const int b = it & 1;
                if (!mbar_wait(&o_full[b], (it >> 1) & 1)) { fail(); break; }
                if (tid == 384) LA_TL(11, it);
                tc_fence_after();
                const int t0 = (c_begin + it) * C;
                const int row = wq * 32 + lane;
                const uint32_t tO = tmem + lane_base + Cfg::COL_O + b * NA;
                float o[48];
                tmem_ld16(tO + DV, o + 32);          // den in column 64
                tmem_ld16(tO, o);
                tmem_ld16(tO + 16, o + 16);
                tmem_ld_wait();
                const float den0 = o[32];
                const float inv = 1.f / den0;
                __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) + ((size_t)bh * N + t0 + row) * DV;
                const bool valid = t0 + row < N;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (half == 1) {
                        tmem_ld16(tO + 32, o);
                        tmem_ld16(tO + 48, o + 16);
                        tmem_ld_wait();
                    }
                    if (valid) {
#pragma unroll
                        for (int c0 = 0; c0 < 32; c0 += 8)
                            *reinterpret_cast<uint4 *>(orow + half * 32 + c0) =
                                make_uint4(pack_bf16(o[c0] * inv, o[c0 + 1] * inv), pack_bf16(o[c0 + 2] * inv, o[c0 + 3] * inv),
                                           pack_bf16(o[c0 + 4] * inv, o[c0 + 5] * inv), pack_bf16(o[c0 + 6] * inv, o[c0 + 7] * inv));
                    }
                }
                if (valid && p.den_out) p.den_out[(size_t)bh * N + t0 + row] = den0;
                tc_fence_before();
                __syncwarp();
                if (tid == 384) LA_TL(12, it);
                if (lane == 0) mbar_arrive(&o_free[b]);
            }
            // final state of the sequence (last segment only): S after the last chunk
            if (seg == p.P - 1 && (p.s_out || p.z_out) && !*abort_flag) {
#pragma unroll 1
                for (int c0 = 0; c0 < NA; c0 += 16) {
                    float v[16];
                    tmem_ld16(tS + c0, v);
                    tmem_ld_wait();
                    if (!frow) continue;
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int col = c0 + e;
                        if (col < DV) {
                            if (p.s_out) p.s_out[((size_t)bh * FP + f) * DV + col] = v[e];
                        } else if (col == DV && p.z_out) {
                            p.z_out[(size_t)bh * FP + f] = v[e];
                        }
                    }
                }
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
                        tmem_ld16(tS + c0, d);
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
