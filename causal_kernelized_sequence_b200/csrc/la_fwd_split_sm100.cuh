// la_fwd_split_sm100.cuh -- chunk-parallel forward for the elu(x)+1 map with
// d_qk = d_v = 64 (bf16 I/O), in two launches, on tcgen05 tensor cores.
//
// Same mathematics as la_prefill_sm100.cuh (BASED page, Knowl 3 parallel
// form, computed chunk by chunk as Knowl 5 describes: a masked quadratic term
// inside each 128-token chunk plus the product with the state of the earlier
// chunks).  What changes is how the state reaches each chunk.  The T chunks of
// all heads, in (head, chunk) order, are cut into G contiguous ranges, one
// per block, G <= 148 (at most 16 ranges per head).
//
//   fwd_split_state_kernel  Per chunk t of its range: phi(K_t) in place on the
//       TMA-loaded K tile (stored to the workspace, swizzled, for the second
//       launch), dS_t = phi(K_t)^T V_aug,t on the tensor cores, and the
//       running sum L of the dS of the earlier chunks of the same head inside
//       the range, written as a bf16 [64 x 80] tile in the layout of an MMA
//       operand: the snapshot of chunk t+1.  It also writes the sum over the
//       range's last head segment (what later ranges of that head need), and
//       the final state of heads that end inside the range.
//   fwd_split_out_kernel  Every chunk is independent.  A block first adds the
//       aggregates of the earlier ranges of its first head into the carry
//       state C (fp32, then one bf16 tile).  Then, per chunk:
//         MMA1  A = phi(Q) phi(K)^T           (phi(Q) in TMEM, phi(K) in smem)
//         mask  P = bf16(A masked to j <= i)  (in place in TMEM)
//         MMA2  O = P V_aug + phi(Q) C + phi(Q) L_t   -> y = O[:, :64] / O[:, 64]
//
// V_aug = [V | 1 | 0 ...] (80 columns), so state [S | z] and output
// [num | den] come out of the same MMAs; as an MN-major SW128 operand its
// second 64-column atom is one constant ones tile shared by every stage.  No
// step waits on another chunk of the same launch, so the roles of a block
// overlap consecutive chunks freely.  phi(K) tiles, snapshots and aggregates
// are written by the first launch and read by the second one from L2.  phi(Q)
// never returns to shared memory: it is formed from the TMA-loaded Q tile and
// stored to TMEM as the A operand of MMA1 and MMA2, and the Q tile is
// released as soon as it has been read.  elu(x)+1 is bound by the special
// function unit (one packed exp2 per two features); each launch forms it once
// per feature.
//
// Every mbarrier wait is bounded (2 s); on expiry a block records a timeout in
// the status word, stops issuing work, frees its TMEM and exits.
#pragma once

#include "la_device.cuh"
#include "la_prefill_sm100.cuh"
#include "sm100.cuh"

namespace la {

struct SplitCfg64 {
    static constexpr int C = 128, D = 64, DV = 64, NA = 80;
    static constexpr int TILE = C * D * 2;                 // 16 KB: a Q, K, phi(K) or V tile (SW128)
    static constexpr int ONES = C * 128;                   // 16 KB: second N-atom of V_aug
    static constexpr int SNAP_BLK = D * 32;                // 2 KB: 16 columns x 64 feature rows
    static constexpr int SNAP = (NA / 16) * SNAP_BLK;      // 10 KB: bf16 [64 x 80] state tile
    static constexpr int AGG = D * NA;                     // fp32 values per aggregate
    static constexpr int MAX_PER_HEAD = 16;                // ranges per head at most
    // state launch: ring of [K | V] stages, two snapshot staging tiles
    static constexpr int S_NS = 5;
    static constexpr int S_STAGE = 2 * TILE;
    static constexpr int S_OFF_ONES = S_NS * S_STAGE;
    static constexpr int S_OFF_SNAP = S_OFF_ONES + ONES;
    static constexpr int S_OFF_BAR = S_OFF_SNAP + 2 * SNAP;
    static constexpr int S_SMEM_ALLOC = S_OFF_BAR + 256 + 1024;
    static constexpr int S_THREADS = 448;
    // output launch: ring of Q tiles, ring of [phi(K) | V | snapshot] stages,
    // two output staging tiles
    static constexpr int O_NQ = 2, O_NKV = 3, O_NPQ = 3;
    static constexpr int O_KV_STAGE = 2 * TILE + SNAP;     // 42 KB
    static constexpr int O_OFF_KV = O_NQ * TILE;
    static constexpr int O_OFF_ONES = O_OFF_KV + O_NKV * O_KV_STAGE;
    static constexpr int O_OFF_Y = O_OFF_ONES + ONES;      // 2 x 16 KB, SW128
    static constexpr int O_OFF_CARRY = O_OFF_Y + 2 * TILE;
    static constexpr int O_OFF_BAR = O_OFF_CARRY + SNAP;
    static constexpr int O_SMEM_ALLOC = O_OFF_BAR + 256 + 1024;
    static constexpr int O_THREADS = 576;
    // 2 x 128: scores fp32, then P bf16 packed: keys 0-63 in columns 0-31,
    // keys 64-127 in columns 96-127
    static constexpr int COL_A = 0;
    static constexpr int COL_O = 256;   // 2 x 80
    static constexpr int COL_PQ = 416;  // 3 x 32: phi(Q) bf16 packed
};

struct SplitParams {
    const float *s_in, *z_in;         // nullable: state entering each sequence, [BH][64][64], [BH][64]
    __nv_bfloat16 *o;
    float *den_out, *s_out, *z_out;   // nullable
    uint8_t *phik;                    // [T][TILE] phi(K) tiles, swizzled as in shared memory
    uint8_t *snap;                    // [T][SNAP] local state before each chunk
    float *agg;                       // [G][2][AGG]: last segment's sum; first segment's sum
    long long T;                      // chunks of all heads
    int N, nc, G;
};

// Optional timeline for profiling builds that define LA_TIMELINE (compiled
// out otherwise): clock64 at role events of block 0 per chunk, and the
// global-timer start and end of every block.
#ifdef LA_TIMELINE
__device__ long long g_tl_split[2][16][64];
__device__ long long g_tl_blocks[2][160][2];
#define LA_TLS(k_, ev, it_)                                                                 \
    do {                                                                                    \
        if (blockIdx.x == 0 && (it_) >= 0 && (it_) < 64) g_tl_split[k_][ev][(it_)] = clock64(); \
    } while (0)
#define LA_TLB(k_, which)                                                                   \
    do {                                                                                    \
        if (threadIdx.x == 0 && blockIdx.x < 160) {                                         \
            long long t_;                                                                   \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                         \
            g_tl_blocks[k_][blockIdx.x][which] = t_;                                        \
        }                                                                                   \
    } while (0)
#else
#define LA_TLS(k_, ev, it_) do { } while (0)
#define LA_TLB(k_, which) do { } while (0)
#endif

namespace split_detail {

// First chunk of range k of G over T chunks.
__host__ __device__ __forceinline__ long long range_begin(long long T, int G, int k)
{
    return (T * (long long)k) / G;
}

__device__ __forceinline__ uint4 elu1_x8(uint4 r)
{
    using namespace fwd_detail;
    return make_uint4(elu1_bf16x2(r.x), elu1_bf16x2(r.y), elu1_bf16x2(r.z), elu1_bf16x2(r.w));
}

// Row r (of 128) of the ones atom: an SW128 row whose column 0 is 1.
__device__ __forceinline__ void write_ones_row(uint8_t *atom, int r)
{
    using namespace fwd_detail;
    uint4 *row = reinterpret_cast<uint4 *>(atom + r * 128);
#pragma unroll
    for (int c = 0; c < 8; ++c)
        row[c] = (c == (r & 7)) ? make_uint4(pack_bf16(1.f, 0.f), 0u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
}

// The range of block kb: first chunk tb, its head h0 and chunk c0 within
// the head, and the chunk count.
struct Range {
    long long tb;
    int nit, h0, c0;
    __device__ Range(const SplitParams &p, int kb)
    {
        tb = range_begin(p.T, p.G, kb);
        nit = (int)(range_begin(p.T, p.G, kb + 1) - tb);
        h0 = (int)(tb / p.nc);
        c0 = (int)(tb - (long long)h0 * p.nc);
    }
    // head and chunk-in-head of the range's chunk `it`
    __device__ __forceinline__ void at(int it, int nc, int &h, int &c) const
    {
        const int x = c0 + it;
        h = h0 + x / nc;
        c = x % nc;
    }
};

}  // namespace split_detail

// ---------------------------------------------------------------- state launch
__global__ void __launch_bounds__(SplitCfg64::S_THREADS, 1)
fwd_split_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const SplitParams p)
{
    using namespace sm100;
    using namespace fwd_detail;
    using namespace split_detail;
    using Cfg = SplitCfg64;
    constexpr int C = Cfg::C, NA = Cfg::NA, DV = Cfg::DV, NS = Cfg::S_NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::S_OFF_BAR);
    uint64_t *full = bars;                 // [NS] K and V landed
    uint64_t *stage_free = bars + NS;      // [NS] MMA3 done and phi(K) stored out
    uint64_t *phi_done = bars + 2 * NS;    // [NS] phi(K) in place (8 warps)
    uint64_t *ds_full = bars + 3 * NS;     // [2]
    uint64_t *ds_free = bars + 3 * NS + 2; // [2] (4 warps)
    uint64_t *sn_full = bars + 3 * NS + 4; // [2] snapshot staged (4 warps)
    uint64_t *sn_free = bars + 3 * NS + 6; // [2] snapshot staging tile read by its store
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * NS + 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 3 * NS + 9);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kb = blockIdx.x;
    const Range rg(p, kb);
    const int nit = rg.nit, nc = p.nc, N = p.N;
    const bool carry_in = rg.c0 != 0;
    const int first_len = min(nit, nc - rg.c0);

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&stage_free[s], 1);
            mbar_init(&phi_done[s], 8);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ds_full[b], 1);
            mbar_init(&ds_free[b], 4);
            mbar_init(&sn_full[b], 4);
            mbar_init(&sn_free[b], 1);
        }
        *abort_flag = 0;
        mbar_init_fence();
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 256);
    if (tid < C) write_ones_row(smem + Cfg::S_OFF_ONES, tid);
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&]() { *abort_flag = 1; };
    // This launch may begin while the previous kernel of the stream finishes
    // (programmatic dependent launch): the setup above overlaps its tail, and
    // nothing is read or written in global memory before that kernel has
    // completed (its writes are then visible; the previous forward's output
    // launch may still read the workspace written below until then).
    grid_dependency_wait();
    // The output launch may take each SM as soon as this block leaves it; it
    // waits for this whole grid before reading anything written here.
    launch_dependents();
    LA_TLB(0, 0);
    if (tid == 0) LA_TLS(0, 15, 0);

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
            for (int it = 0; it < nit && !*abort_flag; ++it) {
                const int s = it % NS;
                if (it >= NS && !mbar_wait(&stage_free[s], ((it / NS) - 1) & 1)) { fail(); break; }
                int h, c;
                rg.at(it, nc, h, c);
                LA_TLS(0, 0, it);
                uint8_t *st = smem + s * Cfg::S_STAGE;
                mbar_arrive_expect_tx(&full[s], 2 * Cfg::TILE);
                tma_load_3d_hint(st, &tm_k, &full[s], 0, c * C, h, drop);           // only phi(K) is reused
                tma_load_3d_hint(st + Cfg::TILE, &tm_v, &full[s], 0, c * C, h, keep);  // read again by the output launch
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------- MMA issuer, phi(K) store
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(64, NA, 1, 1);
            const uint32_t aOnes = smem_addr(smem + Cfg::S_OFF_ONES);
            const uint64_t keep = policy_evict_last();
            for (int it = 0; it < nit && !*abort_flag; ++it) {
                const int s = it % NS, b = it & 1;
                if (!mbar_wait(&full[s], (it / NS) & 1) || !mbar_wait(&phi_done[s], (it / NS) & 1) ||
                    (it >= 2 && !mbar_wait(&ds_free[b], ((it >> 1) - 1) & 1))) {
                    fail();
                    break;
                }
                tc_fence_after();
                LA_TLS(0, 1, it);
                uint8_t *st = smem + s * Cfg::S_STAGE;
                const uint32_t aK = smem_addr(st), aV = aK + Cfg::TILE;
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + b * NA, smem_desc(aK + kk * 2048, C * 128, 1024, kSw128),
                             smem_desc(aV + kk * 2048, aOnes - aV, 1024, kSw128), id_s, kk > 0);
                mma_commit(&ds_full[b]);
                bulk_store_hint(p.phik + (size_t)(rg.tb + it) * Cfg::TILE, st, Cfg::TILE, keep);
                bulk_commit();
                // Free the previous chunk's stage once its phi(K) store has read it
                // (every bulk group but this chunk's has been read), not this one's:
                // the issue of the next chunk's MMA does not wait for the store.
                // The commit also covers this chunk's MMA, issued after the previous
                // one's; the range's last stage is never needed again.
                if (it >= 1) {
                    bulk_wait_read_le1();
                    mma_commit(&stage_free[(it - 1) % NS]);
                }
            }
            asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        }
    } else if (warp < 10) {
        // ------------------------------------------------------- phi(K)
        // elu(x)+1 in place on the K tile; 256 threads, 16-byte piece
        // e = pt + 256 j (j < 4) is row e / 8, columns 8 (e % 8) .. +7 (a warp
        // covers 4 whole swizzled rows: no bank conflicts).  Key rows past N
        // are zeroed so they add nothing.
        const int pt = tid - 64;
        for (int it = 0; it < nit && !*abort_flag; ++it) {
            const int s = it % NS;
            if (!mbar_wait(&full[s], (it / NS) & 1)) { fail(); break; }
            if (pt == 0) LA_TLS(0, 2, it);
            int h, c;
            rg.at(it, nc, h, c);
            const uint32_t tile = smem_addr(smem + s * Cfg::S_STAGE);
            uint4 r[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int e = pt + 256 * j;
                r[j] = lds128(tile + sw128_off(e >> 3, (e & 7) * 8));
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int e = pt + 256 * j;
                sts128(tile + sw128_off(e >> 3, (e & 7) * 8),
                       (c * C + (e >> 3) < N) ? elu1_x8(r[j]) : make_uint4(0u, 0u, 0u, 0u));
            }
            fence_proxy_async();
            __syncwarp();
            if (pt == 0) LA_TLS(0, 3, it);
            if (lane == 0) mbar_arrive(&phi_done[s]);
        }
    } else {
        // ------------------------------------------------------- running state
        // M = 64 TMEM layout: feature row f in lane 32 (f / 16) + f % 16.
        const int wq = warp & 3;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const int f = wq * 16 + lane;
        const bool frow = lane < 16;
        const uint64_t keep = policy_evict_last();
        int ns = 0;   // snapshots written so far (the same count in all four warps)
        float run[NA];
#pragma unroll
        for (int e = 0; e < NA; ++e) run[e] = 0.f;
        // bf16 copy of `run` as the snapshot of range chunk j, in the MMA operand
        // layout: staged in shared memory (double-buffered), then one bulk store
        // by thread 320
        auto write_snap = [&](int j) -> bool {
            const int sb = ns & 1;
            if (ns >= 2 && !mbar_wait(&sn_free[sb], ((ns >> 1) - 1) & 1)) return false;
            const uint32_t stg = smem_addr(smem + Cfg::S_OFF_SNAP + sb * Cfg::SNAP);
            if (frow) {
#pragma unroll
                for (int q = 0; q < NA / 8; ++q)
                    sts128(stg + sw32_off(f, 8 * q, 64),
                           make_uint4(pack_bf16(run[8 * q], run[8 * q + 1]), pack_bf16(run[8 * q + 2], run[8 * q + 3]),
                                      pack_bf16(run[8 * q + 4], run[8 * q + 5]), pack_bf16(run[8 * q + 6], run[8 * q + 7])));
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sn_full[sb]);
            if (tid == 320) {
                if (!mbar_wait(&sn_full[sb], (ns >> 1) & 1)) return false;
                bulk_store_hint(p.snap + (size_t)(rg.tb + j) * Cfg::SNAP, smem + Cfg::S_OFF_SNAP + sb * Cfg::SNAP, Cfg::SNAP,
                                keep);
                bulk_commit();
                bulk_wait_read_le1();   // the previous snapshot's store has read its tile
                if (ns >= 1) mbar_arrive(&sn_free[sb ^ 1]);
            }
            ++ns;
            return true;
        };
        for (int it = 0; it < nit && !*abort_flag; ++it) {
            const int b = it & 1;
            int h, c;
            rg.at(it, nc, h, c);
            if (c == 0) {
                // a head opens: its entering state (zero unless given)
#pragma unroll
                for (int e = 0; e < NA; ++e) run[e] = 0.f;
                if (p.s_in && frow) {
#pragma unroll
                    for (int e = 0; e < DV; ++e) run[e] = p.s_in[((size_t)h * 64 + f) * DV + e];
                    run[DV] = p.z_in[(size_t)h * 64 + f];
                }
                if (p.s_in && !write_snap(it)) { fail(); break; }   // S_snap of this chunk
            }
            if (!mbar_wait(&ds_full[b], (it >> 1) & 1)) { fail(); break; }
            __syncwarp();
            if (tid == 320) LA_TLS(0, 4, it);
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < NA; c0 += 16) {
                float d[16];
                tmem_ld16(tmem + lane_base + b * NA + c0, d);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) run[c0 + e] += d[e];
            }
            tc_fence_before();
            __syncwarp();
            if (tid == 320) LA_TLS(0, 5, it);
            if (lane == 0) mbar_arrive(&ds_free[b]);
            const bool head_end = c == nc - 1, last = it == nit - 1;
            if (!head_end && !last) {
                if (!write_snap(it + 1)) { fail(); break; }   // local state before chunk it+1
                continue;
            }
            if (!frow) continue;
            if (head_end && carry_in && it < first_len) {
                // the head's final state still lacks the carry: left to the output launch
                if (p.s_out || p.z_out) {
                    float4 *dst = reinterpret_cast<float4 *>(p.agg + ((size_t)kb * 2 + 1) * Cfg::AGG + f * NA);
#pragma unroll
                    for (int j = 0; j < NA / 4; ++j)
                        dst[j] = make_float4(run[4 * j], run[4 * j + 1], run[4 * j + 2], run[4 * j + 3]);
                }
            } else if (head_end) {
                if (p.s_out) {
                    float4 *dst = reinterpret_cast<float4 *>(p.s_out + ((size_t)h * 64 + f) * DV);
#pragma unroll
                    for (int j = 0; j < DV / 4; ++j)
                        dst[j] = make_float4(run[4 * j], run[4 * j + 1], run[4 * j + 2], run[4 * j + 3]);
                }
                if (p.z_out) p.z_out[(size_t)h * 64 + f] = run[DV];
            } else {
                // range ends inside a head: the later ranges of the head add this in
                float4 *dst = reinterpret_cast<float4 *>(p.agg + (size_t)kb * 2 * Cfg::AGG + f * NA);
#pragma unroll
                for (int j = 0; j < NA / 4; ++j)
                    dst[j] = make_float4(run[4 * j], run[4 * j + 1], run[4 * j + 2], run[4 * j + 3]);
            }
        }
    }
    if (tid == 320) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) LA_TLS(0, 15, 1);
    LA_TLB(0, 1);
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// --------------------------------------------------------------- output launch
__global__ void __launch_bounds__(SplitCfg64::O_THREADS, 1)
fwd_split_out_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_o, const SplitParams p)
{
    using namespace sm100;
    using namespace fwd_detail;
    using namespace split_detail;
    using Cfg = SplitCfg64;
    constexpr int C = Cfg::C, NA = Cfg::NA, DV = Cfg::DV, NQ = Cfg::O_NQ, NKV = Cfg::O_NKV, NPQ = Cfg::O_NPQ;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::O_OFF_BAR);
    uint64_t *q_full = bars;                // [NQ] Q tile landed
    uint64_t *q_free = q_full + NQ;         // [NQ] Q tile read (4 warps)
    uint64_t *kv_full = q_free + NQ;        // [NKV] phi(K), V (+ snapshot) landed
    uint64_t *kv_free = kv_full + NKV;      // [NKV] MMA2 of the stage done
    uint64_t *pq_full = kv_free + NKV;      // [NPQ] phi(Q) in TMEM (4 warps)
    uint64_t *pq_free = pq_full + NPQ;      // [NPQ] MMA2 done with phi(Q)
    uint64_t *a_full = pq_free + NPQ;       // [2] MMA1 done
    uint64_t *p_full = a_full + 2;          // [2] P written (8)
    uint64_t *o_full = a_full + 4;          // [2] MMA2 done
    uint64_t *o_free = a_full + 6;          // [2] O read (4)
    uint64_t *carry_ready = a_full + 8;     // carry tile stored (4)
    uint64_t *y_full = a_full + 9;          // [2] output staging tile written (4)
    uint64_t *y_free = a_full + 11;         // [2] output staging tile read by its store
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(a_full + 13);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(a_full + 14);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kb = blockIdx.x;
    const Range rg(p, kb);
    const int nit = rg.nit, nc = p.nc, N = p.N;
    const bool carry_in = rg.c0 != 0;
    const int first_len = min(nit, nc - rg.c0);

    if (tid == 0) {
        for (int s = 0; s < NQ; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_free[s], 4);
        }
        for (int s = 0; s < NKV; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_free[s], 1);
        }
        for (int s = 0; s < NPQ; ++s) {
            mbar_init(&pq_full[s], 4);
            mbar_init(&pq_free[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&a_full[b], 1);
            mbar_init(&p_full[b], 8);
            mbar_init(&o_full[b], 1);
            mbar_init(&o_free[b], 4);
            mbar_init(&y_full[b], 4);
            mbar_init(&y_free[b], 1);
        }
        mbar_init(carry_ready, 4);
        *abort_flag = 0;
        mbar_init_fence();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_o);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    if (tid < C) write_ones_row(smem + Cfg::O_OFF_ONES, tid);
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&]() { *abort_flag = 1; };
    // local snapshot exists unless the chunk opens a head segment of the range;
    // where a head opens, it exists when the heads start from a given state
    auto has_loc = [&](int it) {
        const bool opens = (rg.c0 + it) % nc == 0;
        return opens ? p.s_in != nullptr : it > 0;
    };
    auto has_carry = [&](int it) { return carry_in && it < first_len; };
    // The next kernel of the stream may take each SM this block leaves; a
    // dependent launch of the state kernel (the next forward) waits for this
    // whole grid before it touches global memory.
    launch_dependents();
    LA_TLB(1, 0);
    if (tid == 0) LA_TLS(1, 15, 0);

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t drop = policy_evict_first();   // every input here is read for the last time
            auto load_q = [&](int it) {
                int h, c;
                rg.at(it, nc, h, c);
                const int sq = it % NQ;
                mbar_arrive_expect_tx(&q_full[sq], Cfg::TILE);
                tma_load_3d_hint(smem + sq * Cfg::TILE, &tm_q, &q_full[sq], 0, c * C, h, drop);
            };
            // Q does not come from the state launch: start on it before waiting
            for (int it = 0; it < nit && it < NQ; ++it) load_q(it);
            grid_dependency_wait();
            for (int it = 0; it < nit && !*abort_flag; ++it) {
                int h, c;
                rg.at(it, nc, h, c);
                const int skv = it % NKV;
                if (it >= NQ) {
                    if (!mbar_wait(&q_free[it % NQ], ((it / NQ) - 1) & 1)) { fail(); break; }
                    load_q(it);
                }
                LA_TLS(1, 0, it);
                if (it >= NKV && !mbar_wait(&kv_free[skv], ((it / NKV) - 1) & 1)) { fail(); break; }
                uint8_t *st = smem + Cfg::O_OFF_KV + skv * Cfg::O_KV_STAGE;
                const bool loc = has_loc(it);
                const size_t t = (size_t)(rg.tb + it);
                mbar_arrive_expect_tx(&kv_full[skv], 2 * Cfg::TILE + (loc ? Cfg::SNAP : 0));
                bulk_load_hint(st, p.phik + t * Cfg::TILE, Cfg::TILE, &kv_full[skv], drop);
                tma_load_3d_hint(st + Cfg::TILE, &tm_v, &kv_full[skv], 0, c * C, h, drop);
                if (loc) bulk_load_hint(st + 2 * Cfg::TILE, p.snap + t * Cfg::SNAP, Cfg::SNAP, &kv_full[skv], drop);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
            const uint32_t id_o = idesc_bf16(128, NA, 0, 1);
            const uint32_t aCarry = smem_addr(smem + Cfg::O_OFF_CARRY);
            const uint32_t aOnes = smem_addr(smem + Cfg::O_OFF_ONES);
            auto issue_x = [&](int it) {
                const int skv = it % NKV, bq = it % NPQ, b = it & 1;
                LA_TLS(1, 13, it);
                tc_fence_after();
                const uint32_t aK = smem_addr(smem + Cfg::O_OFF_KV + skv * Cfg::O_KV_STAGE);
                const uint32_t dA = tmem + Cfg::COL_A + b * 128, tPQ = tmem + Cfg::COL_PQ + bq * 32;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ts(dA, tPQ + kk * 8, smem_desc(aK + kk * 32, 16, 1024, kSw128), id_qk, kk > 0);
                mma_commit(&a_full[b]);
                LA_TLS(1, 1, it);
            };
            auto issue_y = [&](int it) {
                const int skv = it % NKV, bq = it % NPQ, b = it & 1;
                LA_TLS(1, 10, it);
                tc_fence_after();
                const uint32_t aStage = smem_addr(smem + Cfg::O_OFF_KV + skv * Cfg::O_KV_STAGE);
                const uint32_t aV = aStage + Cfg::TILE, aL = aStage + 2 * Cfg::TILE;
                const uint32_t tP = tmem + Cfg::COL_A + b * 128, tPQ = tmem + Cfg::COL_PQ + bq * 32;
                const uint32_t dO = tmem + Cfg::COL_O + b * NA;
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16_ts(dO, tP + (kk < 4 ? kk * 8 : 96 + (kk - 4) * 8),
                                smem_desc(aV + kk * 2048, aOnes - aV, 1024, kSw128), id_o, kk > 0);
                LA_TLS(1, 11, it);
                if (has_carry(it))
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(dO, tPQ + kk * 8, smem_desc(aCarry + kk * 512, Cfg::SNAP_BLK, 256, kSw32), id_o,
                                    true);
                if (has_loc(it))
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(dO, tPQ + kk * 8, smem_desc(aL + kk * 512, Cfg::SNAP_BLK, 256, kSw32), id_o, true);
                LA_TLS(1, 12, it);
                mma_commit(&o_full[b]);
                mma_commit(&kv_free[skv]);
                mma_commit(&pq_free[bq]);
                LA_TLS(1, 2, it);
            };
            auto x_ready = [&](int it) {
                return mbar_test(&kv_full[it % NKV], (it / NKV) & 1) && mbar_test(&pq_full[it % NPQ], (it / NPQ) & 1);
            };
            auto y_ready = [&](int it) {
                const int b = it & 1;
                return mbar_test(&p_full[b], (it >> 1) & 1) && (it < 2 || mbar_test(&o_free[b], ((it >> 1) - 1) & 1)) &&
                       (!has_carry(it) || mbar_test(carry_ready, 0));
            };
            // Issue whichever of Y(ny) (output of the oldest pending chunk) and
            // X(nx) (scores of the next one) has its inputs ready, preferring Y;
            // X(nx) reuses the score buffer of chunk nx-2, so nx <= ny + 1.
            int nx = 0, ny = 0;
            bool ok = true;
            uint64_t t_last;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_last));
            while (ny < nit && ok && !*abort_flag) {
                bool progress = false;
                if (ny < nx && y_ready(ny)) {
                    issue_y(ny++);
                    progress = true;
                } else if (nx < nit && nx <= ny + 1 && x_ready(nx)) {
                    issue_x(nx++);
                    progress = true;
                }
                if (progress) {
                    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_last));
                } else {
                    uint64_t t;
                    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
                    if (t - t_last > 2000000000ull) {
                        report(kStatusTimeout);
                        ok = false;
                    }
                    __nanosleep(20);   // leave issue slots to the warps sharing this SMSP
                }
            }
            if (!ok) fail();
        }
    } else if (warp < 6) {
        // ------------------------------------------------------- phi(Q) -> TMEM
        // Thread = query row = TMEM lane: the row is read from the swizzled Q
        // tile (conflict-free), phi is applied in registers and the 64
        // features go to TMEM as the A operand of MMA1 and MMA2.
        const int wq = warp & 3, row = wq * 32 + lane;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        for (int it = 0; it < nit && !*abort_flag; ++it) {
            const int sq = it % NQ, bq = it % NPQ;
            if (!mbar_wait(&q_full[sq], (it / NQ) & 1)) { fail(); break; }
            const uint32_t tile = smem_addr(smem + sq * Cfg::TILE);
            uint4 r[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) r[j] = lds128(tile + sw128_off(row, 8 * j));
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_free[sq]);
            uint32_t w[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 v = elu1_x8(r[j]);
                w[4 * j] = v.x;
                w[4 * j + 1] = v.y;
                w[4 * j + 2] = v.z;
                w[4 * j + 3] = v.w;
            }
            if (it >= NPQ && !mbar_wait(&pq_free[bq], ((it / NPQ) - 1) & 1)) { fail(); break; }
            tc_fence_after();
            tmem_st32(tmem + lane_base + Cfg::COL_PQ + bq * 32, w);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (tid == 64) LA_TLS(1, 3, it);
            if (lane == 0) mbar_arrive(&pq_full[bq]);
        }
    } else {
        // --------------------------------------- carry (warps 10-17), then mask / output
        const int wq = warp & 3;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        if (carry_in && warp >= 14) {
            // C = sum of the aggregates of the earlier ranges of this head (ranges
            // jlo .. kb-1), fp32, then one bf16 tile; each of the 128 output
            // threads owns 40 of the 64 x 80 values (10 float4 at pt + 128 m).
            grid_dependency_wait();
            const int pt = tid - 448;
            const long long head0 = rg.tb - rg.c0;
            int jlo = kb - 1;
            while (jlo > 0 && range_begin(p.T, p.G, jlo) > head0) --jlo;
            float4 acc[10];
#pragma unroll
            for (int m = 0; m < 10; ++m) acc[m] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int jb = jlo; jb < kb; ++jb) {
                const float4 *s0 = reinterpret_cast<const float4 *>(p.agg + (size_t)jb * 2 * Cfg::AGG);
                float4 u[10];
#pragma unroll
                for (int m = 0; m < 10; ++m) u[m] = __ldcg(s0 + pt + 128 * m);
#pragma unroll
                for (int m = 0; m < 10; ++m) {
                    acc[m].x += u[m].x;
                    acc[m].y += u[m].y;
                    acc[m].z += u[m].z;
                    acc[m].w += u[m].w;
                }
            }
            const bool fin = (p.s_out || p.z_out) && (first_len < nit || rg.c0 + first_len == nc);
            const float4 *sf = reinterpret_cast<const float4 *>(p.agg + ((size_t)kb * 2 + 1) * Cfg::AGG);
#pragma unroll
            for (int m = 0; m < 10; ++m) {
                const int e4 = pt + 128 * m, f = (4 * e4) / NA, col = (4 * e4) % NA;   // 4 values of row f
                const float4 v = acc[m];
                const uint32_t a = smem_addr(smem + Cfg::O_OFF_CARRY) + sw32_off(f, col, 64);
                asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(pack_bf16(v.x, v.y)),
                             "r"(pack_bf16(v.z, v.w))
                             : "memory");
                if (fin) {
                    // final state of the head = carry + the first segment's own sum
                    const float4 u = __ldcg(sf + e4);
                    const float fs[4] = {v.x + u.x, v.y + u.y, v.z + u.z, v.w + u.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if (col + e < DV) {
                            if (p.s_out) p.s_out[((size_t)rg.h0 * 64 + f) * DV + col + e] = fs[e];
                        } else if (col + e == DV && p.z_out) {
                            p.z_out[(size_t)rg.h0 * 64 + f] = fs[e];
                        }
                    }
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (tid == 512) LA_TLS(1, 9, 0);
            if (lane == 0) mbar_arrive(carry_ready);
        }
        if (warp < 14) {
        // ---------------------------------------------------------------- mask
        // Warps 6-9 take keys 0-63 (P packed in place into columns 0-31), warps
        // 10-13 keys 64-127 (P into columns 96-127, the last 32 keys first), so
        // the two warps of a lane quarter never touch each other's columns.
        const int i = wq * 32 + lane, hf = (warp - 6) >> 2;
        for (int it = 0; it < nit && !*abort_flag; ++it) {
            const int b = it & 1;
            if (!mbar_wait(&a_full[b], (it >> 1) & 1)) { fail(); break; }
            if (tid == 384) LA_TLS(1, 5, it);
            tc_fence_after();
            const uint32_t tA = tmem + lane_base + Cfg::COL_A + b * 128;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int j0 = hf ? 96 - 32 * q : 32 * q;           // key block
                const uint32_t dst = hf ? tA + 112 - 16 * q : tA + 16 * q;
                uint32_t pk[16];
                if (wq * 32 + 31 < j0) {
                    // every key of this block is later than every query of the warp
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                } else {
                    float a[32];
                    tmem_ld32(tA + j0, a);
                    tmem_ld_wait();
                    if (wq * 32 >= j0 + 31) {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) pk[e / 2] = pack_bf16(a[e], a[e + 1]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; e += 2)
                            pk[e / 2] = pack_bf16((j0 + e <= i) ? a[e] : 0.f, (j0 + e + 1 <= i) ? a[e + 1] : 0.f);
                    }
                }
                tmem_st16(dst, reinterpret_cast<const float *>(pk));
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (tid == 384) LA_TLS(1, 6, it);
            if (lane == 0) mbar_arrive(&p_full[b]);
        }
        } else {
        // -------------------------------------------------------------- output
        // y = num / den per row into an SW128 staging tile (double-buffered),
        // then one TMA store of the chunk by thread 448 (rows past N are not
        // written); den straight to global memory.
        const int row = wq * 32 + lane;
        const bool storer = tid == 448;
        const uint64_t drop = policy_evict_first();
        for (int it = 0; it < nit && !*abort_flag; ++it) {
            const int b = it & 1;
            if (!mbar_wait(&o_full[b], (it >> 1) & 1)) { fail(); break; }
            __syncwarp();
            if (tid == 512) LA_TLS(1, 7, it);
            tc_fence_after();
            int h, c;
            rg.at(it, nc, h, c);
            const int tok = c * C + row;
            const uint32_t tO = tmem + lane_base + Cfg::COL_O + b * NA;
            float o[48];
            tmem_ld16(tO + DV, o + 32);   // den in column 64
            tmem_ld16(tO, o);
            tmem_ld16(tO + 16, o + 16);
            tmem_ld_wait();
            const float den0 = o[32];
            const float inv = 1.f / den0;
            // the store of chunk it-2 has finished reading this staging tile
            if (it >= 2 && !mbar_wait(&y_free[b], ((it >> 1) - 1) & 1)) { fail(); break; }
            const uint32_t ytile = smem_addr(smem + Cfg::O_OFF_Y + b * Cfg::TILE);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                if (half == 1) {
                    tmem_ld16(tO + 32, o);
                    tmem_ld16(tO + 48, o + 16);
                    tmem_ld_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&o_free[b]);
                }
#pragma unroll
                for (int c0 = 0; c0 < 32; c0 += 8)
                    sts128(ytile + sw128_off(row, half * 32 + c0),
                           make_uint4(pack_bf16(o[c0] * inv, o[c0 + 1] * inv), pack_bf16(o[c0 + 2] * inv, o[c0 + 3] * inv),
                                      pack_bf16(o[c0 + 4] * inv, o[c0 + 5] * inv), pack_bf16(o[c0 + 6] * inv, o[c0 + 7] * inv)));
            }
            if (tok < N && p.den_out) p.den_out[(size_t)h * N + tok] = den0;
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&y_full[b]);
            if (storer) {
                if (!mbar_wait(&y_full[b], (it >> 1) & 1)) { fail(); break; }
                tma_store_3d_hint(&tm_o, smem + Cfg::O_OFF_Y + b * Cfg::TILE, 0, c * C, h, drop);
                bulk_commit();
                // the store of chunk it-1 has read its tile: free it for chunk it+1
                bulk_wait_read_le1();
                if (it >= 1) mbar_arrive(&y_free[b ^ 1]);
            }
            if (tid == 512) LA_TLS(1, 8, it);
        }
        if (storer) bulk_wait_all();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) LA_TLS(1, 15, 1);
    LA_TLB(1, 1);
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace la
