// la_swa.cuh -- causal sliding-window softmax attention: prefill on the
// tensor cores, exact fp32 CUDA-core kernels, and the w-token key/value cache
// of generation.
//
// The method ("Simple linear attention language models balance the
// recall-throughput tradeoff", Knowl 4): query i attends only to keys
// max(0, i-w+1) .. i,
//     o_i = sum_j softmax_j(s_ij) v_j,   s_ij = q_i.k_j / sqrt(dqk),
// with w a small multiple of 16; generation keeps the last w keys and values
// (Knowl 4 and the sliding-window generation kernel of Knowl 5).
//
// Tensor-core prefill (bf16, dqk = dv = 64, w a multiple of 16 up to 128):
// one CTA of 256 threads (two per query row) per 128-query tile, persistent
// over tiles.
//   TMA     Q tile [128 x 64] and K, V spans [128 + w x 64] starting w keys
//           before the tile (a negative start reads zeros), SW128.
//   MMA1    S = Q K^T  [128 x (128 + w)] fp32 -> TMEM.
//   softmax the two threads of row i read the band of the row (columns
//           i+1 .. i+w of the span, the keys t0+i-w+1 .. t0+i) in two parts,
//           combine max and sum through shared memory, and write P (bf16,
//           zero off the band) over the Q/K buffer, which MMA1 no longer needs.
//   MMA2    O = P V  [128 x 64] -> TMEM; then o = O / rowsum, bf16.
// The next tile's loads are issued as soon as MMA2 completes, under the
// epilogue.  For w <= 64 a CTA takes 256 TMEM columns and 80 KB of shared
// memory, so two CTAs share an SM and overlap each other's steps.
#pragma once

#include "la_device.cuh"
#include "la_prefill_sm100.cuh"
#include "sm100.cuh"

namespace la {

template <int W_>
struct SwaCfg {
    static constexpr int W = W_;
    static constexpr int C = 128;                    // queries per tile
    static constexpr int D = 64;                     // dqk = dv
    static constexpr int KW = C + W;                 // keys spanned by a tile
    static constexpr int Q_TILE = C * 128;           // 128 rows x 128 B
    static constexpr int KV_TILE = KW * 128;
    static constexpr int P_TILE = ((KW + 63) / 64) * C * 128;   // K-major SW128 blocks of 64 keys
    static constexpr int QK_BYTES = Q_TILE + KV_TILE;
    static constexpr int REGION_A = ((QK_BYTES > P_TILE ? QK_BYTES : P_TILE) + 1023) / 1024 * 1024;
    static constexpr int OFF_Q = 0, OFF_K = Q_TILE, OFF_P = 0;
    static constexpr int OFF_V = REGION_A;
    static constexpr int OFF_BAR = OFF_V + (KV_TILE + 1023) / 1024 * 1024;
    static constexpr int OFF_RED = OFF_BAR + 64;     // row max and row sum of each half: 4 x 128 floats
    static constexpr int OFF_Y = (OFF_RED + 4 * C * 4 + 1023) / 1024 * 1024;   // o tile (SW128), stored by TMA
    static constexpr int SMEM = OFF_Y + C * 128;
    static constexpr int COL_S = 0;
    static constexpr int COL_O = (KW + 31) / 32 * 32;
    static constexpr int TMEM_COLS = COL_O + D <= 256 ? 256 : 512;
    // Residency follows TMEM (512 columns per SM): at most two CTAs of 256
    // columns, or one of 512, per SM.  A shared-memory floor enforces it, so no
    // CTA's allocation waits on a persistent neighbour.
    static constexpr int SMEM_FLOOR = TMEM_COLS == 256 ? 80 * 1024 : 120 * 1024;
    static constexpr int SMEM_ALLOC = SMEM + 1024 > SMEM_FLOOR ? SMEM + 1024 : SMEM_FLOOR;
    static constexpr int NCOL = 32 + W;              // span columns a warp's rows can touch
    // two threads per query row (warps w and w + 4 reach the same TMEM lanes):
    // the first takes H0 of those columns, the second the other H1
    static constexpr int H0 = 16 * ((NCOL + 31) / 32), H1 = NCOL - H0;
    static constexpr int THREADS = 256;
    static constexpr int MIN_BLOCKS = TMEM_COLS == 256 ? 2 : 1;
    static_assert(W % 16 == 0 && W >= 16 && W <= 128, "window: a multiple of 16 up to 128");
    static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory");
};

struct SwaParams {
    __nv_bfloat16 *o;   // [BH, N, 64]
    float *lse;         // [BH, N] nullable: log-sum-exp of the scaled scores
    int N, BH, tiles_per_bh;
    float scale_log2;   // log2(e) / sqrt(dqk)
    float scale;        // 1 / sqrt(dqk)
};

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, Cfg::MIN_BLOCKS)
swa_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, const SwaParams p)
{
    using namespace sm100;
    using namespace fwd_detail;
    constexpr int C = Cfg::C, W = Cfg::W, KW = Cfg::KW;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *load_bar = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *mma_bar = load_bar + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(load_bar + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(load_bar + 3);

    // Launched as a programmatic dependent: nothing in global memory is read
    // or written before the previous kernel of the stream has completed; the
    // next one may then take the SMs this grid leaves.
    grid_dependency_wait();
    launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, hh = warp >> 2, row = wq * 32 + lane;   // TMEM lane quadrant, row half
    const int ntiles = p.BH * p.tiles_per_bh;
    float *red_m = reinterpret_cast<float *>(smem + Cfg::OFF_RED);   // [2][C] row max per half
    float *red_s = red_m + 2 * C;                                    // [2][C] row sum per half

    if (tid == 0) {
        mbar_init(load_bar, 1);
        mbar_init(mma_bar, 1);
        *abort_flag = 0;
        mbar_init_fence();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_o);
    }
    if (warp == 0) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const uint32_t aQ = smem_addr(smem + Cfg::OFF_Q), aK = smem_addr(smem + Cfg::OFF_K);
    const uint32_t aV = smem_addr(smem + Cfg::OFF_V), aP = smem_addr(smem + Cfg::OFF_P);

    auto issue_loads = [&](int tile) {
        const int bh = tile / p.tiles_per_bh, t0 = (tile - bh * p.tiles_per_bh) * C;
        mbar_arrive_expect_tx(load_bar, Cfg::Q_TILE + 2 * Cfg::KV_TILE);
        tma_load_3d(smem + Cfg::OFF_Q, &tm_q, load_bar, 0, t0, bh);
        tma_load_3d(smem + Cfg::OFF_K, &tm_k, load_bar, 0, t0 - W, bh);
        tma_load_3d(smem + Cfg::OFF_V, &tm_v, load_bar, 0, t0 - W, bh);
    };

    uint32_t load_phase = 0, mma_phase = 0;
    bool load_pending = false;   // thread 0: a tile's loads issued and not yet waited for
    // A tile's o goes to the o tile in shared memory and leaves by one TMA store,
    // issued by thread 0 once every thread has passed the next barrier (rows past
    // the slice's end are clipped by the tensor map)
    int y_bh = -1, y_t0 = 0;     // thread 0: the tile whose o waits in the o tile
    auto store_y = [&]() {
        tma_store_3d(&tm_o, smem + Cfg::OFF_Y, 0, y_t0, y_bh);
        bulk_commit();
        y_bh = -1;
    };
    if (tid == 0 && (int)blockIdx.x < ntiles) {
        issue_loads(blockIdx.x);
        load_pending = true;
    }

    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int bh = tile / p.tiles_per_bh, t0 = (tile - bh * p.tiles_per_bh) * C;
        if (!mbar_wait(load_bar, load_phase)) *abort_flag = 1;
        load_phase ^= 1u;
        load_pending = false;
        tc_fence_after();
        // ---- MMA1: S = Q K^T
        if (tid == 0 && !*abort_flag) {
            const uint32_t id = idesc_bf16(128, KW, 0, 0);
#pragma unroll
            for (int kk = 0; kk < Cfg::D / 16; ++kk)
                mma_bf16(tmem + Cfg::COL_S, smem_desc(aQ + kk * 32, 16, 1024, kSw128),
                         smem_desc(aK + kk * 32, 16, 1024, kSw128), id, kk > 0);
            mma_commit(mma_bar);
        }
        if (!mbar_wait(mma_bar, mma_phase)) *abort_flag = 1;
        mma_phase ^= 1u;
        tc_fence_after();

        // ---- softmax over the band of row i: span columns i+1 .. i+W, and
        // only keys at index >= 0 (column >= W - t0).  The two threads of a row
        // take the columns [c0, c0 + nh) of the warp's span (nh = H0 or H1; the
        // guard c < nh is the same across a warp).
        float rowmax, rowsum;
        {
            const int i = row, c_base = wq * 32;
            const int c0 = c_base + (hh ? Cfg::H0 : 0), nh = hh ? Cfg::H1 : Cfg::H0;
            const int lo = max(i + 1, W - t0), hi = i + W;   // inclusive band in span columns
            float sv[Cfg::H0];
#pragma unroll
            for (int c = 0; c < Cfg::H0; c += 16)
                if (c < nh) tmem_ld16(tmem + lane_base + Cfg::COL_S + c0 + c, sv + c);
            tmem_ld_wait();
            float m = -INFINITY;
#pragma unroll
            for (int c = 0; c < Cfg::H0; ++c)
                if (c < nh && c0 + c >= lo && c0 + c <= hi) m = fmaxf(m, sv[c]);
            red_m[hh * C + i] = m;
            __syncthreads();
            if (tid == 0 && y_bh >= 0) store_y();   // the previous tile's o
            rowmax = fmaxf(red_m[i], red_m[C + i]);
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < Cfg::H0; ++c) {
                const float e = (c < nh && c0 + c >= lo && c0 + c <= hi) ? exp2f((sv[c] - rowmax) * p.scale_log2) : 0.f;
                sv[c] = e;
                sum += e;
            }
            red_s[hh * C + i] = sum;
            // P row i over these columns (K-major SW128 blocks of 64 keys), zeros
            // off the warp's span: the first half left of it, the second right of it
#pragma unroll
            for (int c = 0; c < Cfg::H0; c += 8)
                if (c < nh)
                    sts128(aP + sw128_off(i, c0 + c),
                           make_uint4(pack_bf16(sv[c], sv[c + 1]), pack_bf16(sv[c + 2], sv[c + 3]),
                                      pack_bf16(sv[c + 4], sv[c + 5]), pack_bf16(sv[c + 6], sv[c + 7])));
            if (hh == 0)
                for (int col = 0; col < c_base; col += 8) sts128(aP + sw128_off(i, col), make_uint4(0u, 0u, 0u, 0u));
            else
                for (int col = c_base + Cfg::NCOL; col < KW; col += 8)
                    sts128(aP + sw128_off(i, col), make_uint4(0u, 0u, 0u, 0u));
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (*abort_flag) break;

        // ---- MMA2: O = P V   (its epilogue rewrites the o tile: the previous
        // tile's store must have read it)
        if (tid == 0) {
            bulk_wait_read();
            const uint32_t id = idesc_bf16(128, Cfg::D, 0, 1);
#pragma unroll
            for (int kk = 0; kk < KW / 16; ++kk) {
                const uint32_t off = (kk >> 2) * (C * 128) + (kk & 3) * 32;
                mma_bf16(tmem + Cfg::COL_O, smem_desc(aP + off, 16, 1024, kSw128),
                         smem_desc(aV + kk * 2048, Cfg::KV_TILE, 1024, kSw128), id, kk > 0);
            }
            mma_commit(mma_bar);
        }
        if (!mbar_wait(mma_bar, mma_phase)) *abort_flag = 1;
        mma_phase ^= 1u;
        tc_fence_after();
        // the buffers are free: the next tile's loads run under this epilogue
        if (tid == 0 && !*abort_flag && tile + (int)gridDim.x < ntiles) {
            issue_loads(tile + gridDim.x);
            load_pending = true;
        }

        // ---- epilogue: o = O / rowsum (bf16; this thread's 32 of the 64 columns), lse
        {
            const int i = row;
            constexpr int DH = Cfg::D / 2;
            rowsum = red_s[i] + red_s[C + i];   // both halves, written before the barrier above
            float ov[DH];
#pragma unroll
            for (int c = 0; c < DH; c += 16) tmem_ld16(tmem + lane_base + Cfg::COL_O + hh * DH + c, ov + c);
            tmem_ld_wait();
            const float inv = 1.f / rowsum;
#pragma unroll
            for (int c = 0; c < DH; c += 8)
                sts128(smem_addr(smem + Cfg::OFF_Y) + sw128_off(i, hh * DH + c),
                       make_uint4(pack_bf16(ov[c] * inv, ov[c + 1] * inv), pack_bf16(ov[c + 2] * inv, ov[c + 3] * inv),
                                  pack_bf16(ov[c + 4] * inv, ov[c + 5] * inv), pack_bf16(ov[c + 6] * inv, ov[c + 7] * inv)));
            if (t0 + i < p.N && p.lse && hh == 0) p.lse[(size_t)bh * p.N + t0 + i] = rowmax * p.scale + logf(rowsum);
            fence_proxy_async();
            if (tid == 0) {
                y_bh = bh;
                y_t0 = t0;
            }
        }
        tc_fence_before();
    }
    // after an early exit, let this CTA's own copies land before leaving (bounded)
    if (tid == 0 && load_pending) mbar_wait(load_bar, load_phase, 100000000ull);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        if (y_bh >= 0 && !*abort_flag) store_y();   // the last tile's o
        bulk_wait_all();
    }
    if (warp == 0) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

// ---------------------------------------------------------- exact fp32 path

constexpr int kSwaSimtWarps = 8;
constexpr int kSwaMaxWindow = 1024;

// One warp per query row, 8 rows per block.  Scores: lanes over keys (each
// lane a full dot product); output: lanes over value columns.  fp32 FMA and
// expf throughout.  Dynamic shared memory: per warp w scores and dqk floats.
template <typename T>
__global__ void __launch_bounds__(32 * kSwaSimtWarps)
swa_fwd_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, T *__restrict__ o,
                    float *__restrict__ lse, int N, int dqk, int dv, int w, float scale)
{
    extern __shared__ float sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *sc = sm + (size_t)warp * (w + dqk);
    float *qs = sc + w;
    const int rblocks = (N + kSwaSimtWarps - 1) / kSwaSimtWarps;   // grid: (b,h) x row blocks, flattened
    const size_t bh = blockIdx.x / rblocks;
    const int i = (int)(blockIdx.x - bh * rblocks) * kSwaSimtWarps + warp;
    if (i >= N) return;
    const T *qb = q + (bh * N + i) * dqk;
    for (int c = lane; c < dqk; c += 32) qs[c] = ld(qb + c);
    __syncwarp();
    const int j0 = max(0, i - w + 1), n = i - j0 + 1;
    float m = -INFINITY;
    for (int jj = lane; jj < n; jj += 32) {
        const T *kr = k + (bh * N + j0 + jj) * dqk;
        float s = 0.f;
        for (int c = 0; c < dqk; ++c) s = fmaf(qs[c], ld(kr + c), s);
        s *= scale;
        sc[jj] = s;
        m = fmaxf(m, s);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float den = 0.f;
    for (int jj = lane; jj < n; jj += 32) {
        const float e = expf(sc[jj] - m);
        sc[jj] = e;
        den += e;
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    __syncwarp();
    for (int c = lane; c < dv; c += 32) {
        float acc = 0.f;
        for (int jj = 0; jj < n; ++jj) acc = fmaf(sc[jj], ld(v + (bh * N + j0 + jj) * dv + c), acc);
        st(o + (bh * N + i) * dv + c, acc / den);
    }
    if (lse && lane == 0) lse[bh * N + i] = m + logf(den);
}

// ------------------------------------------------------------------ the cache

// k_cache [BH, w, dqk], v_cache [BH, w, dv]: token t of a sequence lives in
// slot t mod w.  Fill from the last min(N, w) tokens of a prefill.
template <typename T>
__global__ void swa_cache_fill_kernel(const T *__restrict__ k, const T *__restrict__ v, T *__restrict__ kc,
                                      T *__restrict__ vc, int N, int dqk, int dv, int w)
{
    const size_t bh = blockIdx.x;
    const int first = max(0, N - w), n = N - first;
    for (int idx = threadIdx.x; idx < n * dqk; idx += blockDim.x) {
        const int t = first + idx / dqk, c = idx % dqk;
        kc[(bh * w + t % w) * dqk + c] = k[(bh * N + t) * dqk + c];
    }
    for (int idx = threadIdx.x; idx < n * dv; idx += blockDim.x) {
        const int t = first + idx / dv, c = idx % dv;
        vc[(bh * w + t % w) * dv + c] = v[(bh * N + t) * dv + c];
    }
}

constexpr int kSwaDecodeThreads = 128;

// One decode step per (b, h): store k, v in slot pos[b] mod w, then attend
// over the min(pos[b] + 1, w) cached tokens (softmax order does not matter).
// Shared memory: w scores, dqk query floats, 4 + 4 reduction floats.
template <typename T>
__global__ void __launch_bounds__(kSwaDecodeThreads)
swa_decode_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, T *__restrict__ y,
                  T *__restrict__ kc, T *__restrict__ vc, const int *__restrict__ pos, int H, int dqk, int dv,
                  int w, float scale)
{
    extern __shared__ float sm[];
    float *sc = sm, *qs = sc + w, *red = qs + dqk;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t bh = blockIdx.x;
    const int b = (int)(bh / H);
    const int t = pos[b];
    if (t < 0) {
        if (tid == 0) report(kStatusCheck);
        return;
    }
    const int slot = t % w, n = min(t + 1, w);
    T *kb = kc + bh * w * dqk, *vb = vc + bh * w * dv;
    for (int c = tid; c < dqk; c += kSwaDecodeThreads) {
        kb[(size_t)slot * dqk + c] = k[bh * dqk + c];
        qs[c] = ld(q + bh * dqk + c);
    }
    for (int c = tid; c < dv; c += kSwaDecodeThreads) vb[(size_t)slot * dv + c] = v[bh * dv + c];
    __syncthreads();
    float m = -INFINITY;
    for (int j = tid; j < n; j += kSwaDecodeThreads) {
        float s = 0.f;
        for (int c = 0; c < dqk; ++c) s = fmaf(qs[c], ld(kb + (size_t)j * dqk + c), s);
        s *= scale;
        sc[j] = s;
        m = fmaxf(m, s);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    float den = 0.f;
    for (int j = tid; j < n; j += kSwaDecodeThreads) {
        const float e = expf(sc[j] - m);
        sc[j] = e;
        den += e;
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    if (lane == 0) red[4 + warp] = den;
    __syncthreads();
    den = (red[4] + red[5]) + (red[6] + red[7]);
    for (int c = tid; c < dv; c += kSwaDecodeThreads) {
        float acc = 0.f;
        for (int j = 0; j < n; ++j) acc = fmaf(sc[j], ld(vb + (size_t)j * dv + c), acc);
        st(y + bh * dv + c, acc / den);
    }
}

// 8 consecutive elements as floats (16-byte loads; rows are 16-byte aligned).
__device__ __forceinline__ void load8(const float *p, float *f)
{
    const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float *f)
{
    fwd_detail::unpack8(*reinterpret_cast<const uint4 *>(p), f);
}
__device__ __forceinline__ void copy8(float *dst, const float *src)
{
    reinterpret_cast<float4 *>(dst)[0] = reinterpret_cast<const float4 *>(src)[0];
    reinterpret_cast<float4 *>(dst)[1] = reinterpret_cast<const float4 *>(src)[1];
}
__device__ __forceinline__ void copy8(__nv_bfloat16 *dst, const __nv_bfloat16 *src)
{
    *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(src);
}

// Decode step for d = dv = 64 and windows up to 64, one 128-thread block per
// (b, h).  Every load is issued up front with 16-byte accesses: thread pair
// (2j, 2j+1) holds key j (one half of d each) and thread (g, c) the value
// columns 8c..8c+7 of keys g, g+16, g+32, g+48.  The new token's k and v
// are read from the inputs, not from its cache slot, so the slot can be
// written without a barrier before the scores.
template <typename T>
__global__ void __launch_bounds__(128, 4)
swa_decode64_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v, T *__restrict__ y,
                    T *__restrict__ kc, T *__restrict__ vc, const int *__restrict__ pos, int H, int w, float scale)
{
    __shared__ float p_s[64];
    __shared__ float part[16][64];
    __shared__ float red[8];
    // Launched as a programmatic dependent: the previous step's cache writes
    // and outputs are complete and visible once this returns; the next step's
    // blocks may then take the SMs this grid leaves.
    sm100::grid_dependency_wait();
    sm100::launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t bh = blockIdx.x;
    const int t = pos[bh / H];
    if (t < 0) {
        if (tid == 0) report(kStatusCheck);
        return;
    }
    const int slot = t % w, n = min(t + 1, w);
    const T *kin = k + bh * 64, *vin = v + bh * 64;
    T *kb = kc + bh * (size_t)w * 64, *vb = vc + bh * (size_t)w * 64;
    // keys
    const int j = tid >> 1, h = tid & 1;
    float kf[32], qf[32];
    const bool kvalid = j < n;
    const T *krow = (j == slot ? kin : kb + (size_t)j * 64) + h * 32;
#pragma unroll
    for (int e = 0; e < 32; e += 8) {
        if (kvalid) load8(krow + e, kf + e);
        load8(q + bh * 64 + h * 32 + e, qf + e);
    }
    // values
    const int g = tid >> 3, c8 = (tid & 7) * 8;
    float vf[4][8];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int jj = g + 16 * r;
        if (jj < n) load8((jj == slot ? vin : vb + (size_t)jj * 64) + c8, vf[r]);
    }
    // the new token into its slot (no thread reads the slot from the cache)
    if (tid < 8) copy8(kb + (size_t)slot * 64 + tid * 8, kin + tid * 8);
    else if (tid < 16) copy8(vb + (size_t)slot * 64 + (tid - 8) * 8, vin + (tid - 8) * 8);
    // scores and softmax
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) s = fmaf(qf[e], kvalid ? kf[e] : 0.f, s);
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s = kvalid ? s * scale : -INFINITY;
    float m = s;
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float e = kvalid ? expf(s - m) : 0.f;
    if (h == 0) p_s[j] = e;
    float den = h == 0 ? e : 0.f;
#pragma unroll
    for (int off = 16; off; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    if (lane == 0) red[4 + warp] = den;
    __syncthreads();
    den = (red[4] + red[5]) + (red[6] + red[7]);
    // outputs: partial sums of 16 key groups, then one column per thread
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int jj = g + 16 * r;
        if (jj < n) {
            const float pj = p_s[jj];
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[c] = fmaf(pj, vf[r][c], acc[c]);
        }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) part[g][c8 + c] = acc[c];
    __syncthreads();
    if (tid < 64) {
        float o = 0.f;
#pragma unroll
        for (int gg = 0; gg < 16; ++gg) o += part[gg][tid];
        st(y + bh * 64 + tid, o / den);
    }
}

}  // namespace la
