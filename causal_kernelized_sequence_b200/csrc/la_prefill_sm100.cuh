// la_prefill_sm100.cuh -- chunked causal linear attention forward on the
// 5th-generation tensor cores (tcgen05 + TMEM), with TMA-staged inputs.
//
// The method (BASED page, Knowl 3 parallel form; Knowl 5 chunked prefill):
// for a chunk c of C = 128 tokens with state (S, z) accumulated over the
// earlier chunks,
//     y_i = [ sum_{j<=i in c} a_ij v_j + phi(q_i) S ] / [ sum_{j<=i} a_ij + phi(q_i).z ],
//     S  += phi(K_c)^T V_c,   z += sum_j phi(k_j).
// The normaliser rides along as an extra value column: V_aug = [V | 1 | 0..0]
// (DV + 16 columns), so S_aug = [S | z] and one accumulator row holds both
// numerator and denominator, rounded identically.
//
// Per chunk (one CTA of 256 worker threads plus one warp whose first thread
// issues the MMAs and the refill loads; token i <-> TMEM lane i, whose row two
// workers share, warps w and w + 4 each taking half of its columns):
//   TMA     Q_c, K_c (SW128, or SW32 for d'=16) and V_c (SW32) into a
//           2-stage ring (d = 128: one stage, with the next chunk's K loaded
//           once MMA1 and MMA3 are done with this one's; the segment pass,
//           which reads only K and V, two).  Rows past the slice's
//           end read as zeros (fixed length) or hold the next packed
//           sequence's tokens; either way they are kept out of the state
//           and out of every stored row.
//   phi     elu(x)+1 applied in place to the Q/K tiles; for the Taylor map
//           the symmetric second-order features (1 + 16 + 136 = 153, padded
//           to 160) are written to separate phi tiles.  phi(q).phi(k) equals
//           1 + q.k/sqrt(d') + (q.k)^2/(2 d') exactly as for the 273-feature
//           map.  The state at the boundary is either expanded back to 273
//           rows or, for the folded map, is these 153 rows as they are.
//   MMA1    A = phi(Q_c) phi(K_c)^T      (Taylor: Q_c K_c^T, then the closed
//           form 1 + s/sqrt(d') + s^2/(2d') in the mask pass)   -> TMEM,
//           with a commit of its own so the mask pass need not wait for MMA3
//   MMA3    S_aug += phi(K_c)^T V_aug   (feature rows in TMEM lanes); issued
//           right after MMA1, or with MMA2 in the gated form, whose phi(K)
//           rows are first scaled by their decay to the chunk's end
//   mask    causal mask j <= i, bf16 -> P tile in shared memory
//   MMA2    O_aug = P V_aug + phi(Q_c) S_snap   (S_snap = bf16 copy of the
//           state entering the chunk)                             -> TMEM
//   out     y = O[:, :DV] / O[:, DV]; S_snap <- bf16(S_aug) for the next chunk.
//
// Long sequences with few heads are split into P segments per head: a first
// kernel computes each segment's state increment (MMA3 only) into the
// caller's workspace; each segment of the main kernel starts from the sum of
// the increments of the segments before it.
#pragma once

#include <type_traits>

#include "la_device.cuh"
#include "sm100.cuh"

namespace la {

template <int DQK_, int DV_, bool TAYLOR_>
struct FwdCfg {
    static constexpr int DQK = DQK_;
    static constexpr int DV = DV_;
    static constexpr bool TAYLOR = TAYLOR_;
    static constexpr int C = 128;                       // tokens per chunk
    static constexpr int NA = DV + 16;                  // value columns + normaliser block
    static constexpr int FSYM = TAYLOR ? 1 + DQK + DQK * (DQK + 1) / 2 : DQK;
    static constexpr int FP = TAYLOR ? 160 : DQK;       // K extent of phi(Q) S_snap
    static constexpr int FT = TAYLOR ? 192 : DQK;       // feature extent of phi tiles
    static constexpr int STAGES = (DQK == 128) ? 1 : 2;
    // State tiles (features in TMEM lanes).  M of each tile:
    static constexpr int NT = TAYLOR ? 2 : 1;
    static __host__ __device__ constexpr int tile_m(int t) { return TAYLOR ? (t == 0 ? 128 : 64) : DQK; }
    static __host__ __device__ constexpr int tile_f0(int t) { return t == 0 ? 0 : 128; }
    // TMEM columns
    static constexpr int COL_O = 0;
    static constexpr int COL_S = (C > NA ? C : NA);
    // Taylor: phi(Q) as bf16 pairs (the A operand of MMA2's state term)
    static constexpr int COL_PQ = COL_S + NT * NA;
    static constexpr int TMEM_USED = COL_PQ + (TAYLOR ? FP / 2 : 0);
    static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;
    // Shared memory (bytes; every region 1024-aligned)
    static constexpr int QK_TILE = TAYLOR ? C * 32 : C * DQK * 2;   // one raw Q or K tile
    static constexpr int V_BLK = C * 32;                            // one 16-column SW32 block
    static constexpr int V_TILE = (DV / 16 + 1) * V_BLK;            // V blocks + ones block
    static constexpr int PHI_TILE = TAYLOR ? C * FT * 2 : 0;
    static constexpr int P_TILE = C * C * 2;
    static constexpr int S_BLK = FP * 32;                           // one 16-column block of S_snap
    static constexpr int S_TILE = (NA / 16) * S_BLK;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + STAGES * QK_TILE;
    static constexpr int OFF_V = OFF_K + STAGES * QK_TILE;
    // Taylor: two phi(K) tiles (phi(Q) lives in TMEM): the next chunk's is built
    // while this chunk's MMA2 runs (ungated full forward)
    static constexpr int OFF_PQ = OFF_V + ((STAGES * V_TILE + 1023) / 1024) * 1024;
    static constexpr int OFF_PK = OFF_PQ + PHI_TILE;
    static constexpr int OFF_P = OFF_PK + PHI_TILE;
    static constexpr int OFF_S = OFF_P + P_TILE;
    static constexpr int OFF_BAR = OFF_S + ((S_TILE + 1023) / 1024) * 1024;
    static constexpr int OFF_G = OFF_BAR + 128;         // gated form: C prefix sums + 4 warp totals
    static constexpr int SMEM = OFF_G + (C + 4) * 4;
    static constexpr int SMEM_ALLOC = SMEM + 1024;      // slack for 1024-byte alignment
    static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory per block");
    static constexpr int TX_BYTES = 2 * C * DQK * 2 + C * DV * 2;
};

struct FwdParams {
    const float *s_in;  // [BH, F, DV] nullable: state entering the sequence
    const float *z_in;  // [BH, F]
    float *s_out;       // [BH, F, DV] nullable
    float *z_out;       // [BH, F] nullable
    // Taylor boundary layout of s_in/z_in/s_out/z_out: 0 = 273 features (row
    // pairs (a,b), (b,a) unfolded), 1 = the 153 folded features, which are
    // the kernel's own rows 0..152.
    int sym_state;
    float *den_out;     // [BH, N] nullable
    float *ws;          // [BH, P, FP, NA] segment increments (P > 1)
    void *o;            // [BH, N, DV] bf16
    int N, P, nchunks, cps;
    // Packed sequences (nullable): sequence n holds tokens cu[n] .. cu[n+1]-1
    // of every head of a [H, T, *] batch; the grid is nseq x H x P blocks and
    // the state slices are (n, h).  N, nchunks and cps are then those of the
    // longest allowed sequence, max_len.
    const int *cu;
    int H, T, max_len;
    float inv_c1, inv_c2;       // Taylor: 1/d'^(1/4), 1/(sqrt(2) sqrt(d'))
    float k1, k2;               // Taylor closed form: 1/sqrt(d'), 1/(2 d')
    // Gated form (nullable): log forget gate g_t per token, at the token's row
    // (row0 + t).  With P > 1 the segment-state launch also writes each
    // segment's summed gate after the increments in ws, and a segment starts
    // from the increments before it, each decayed by the gates after it.
    const float *logdecay;
};

namespace fwd_detail {

// Byte offset of element (row r, column col) inside a tile stored as
// 128-byte swizzled rows (TMA SWIZZLE_128B / UMMA SW128, 64 bf16 per row
// block, 128 rows per block).
__device__ __forceinline__ uint32_t sw128_off(int r, int col)
{
    const int blk = col >> 6, c = (col >> 3) & 7;
    return blk * (128 * 128) + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4) + (col & 7) * 2;
}

// Byte offset of (row r, column col) in a 32-byte swizzled layout made of
// 16-column blocks of `rows` rows each (TMA SWIZZLE_32B / UMMA SW32).
__device__ __forceinline__ uint32_t sw32_off(int r, int col, int rows)
{
    const int blk = col >> 4, c = (col >> 3) & 1;
    return blk * (rows * 32) + (r >> 3) * 256 + (r & 7) * 32 + ((c ^ ((r >> 2) & 1)) << 4) + (col & 7) * 2;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ void unpack8(uint4 u, float *f)
{
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

// elu(x)+1 on two packed bf16 values: max(x,0) + 2^(min(x,0) log2 e).  The
// exponent argument min(x,0) * log2 e is formed with log2 e split into a bf16
// head (1.4453125) and tail (-0.00262451), as fma(n, head, n * tail), so it is
// rounded once; the packed exp2 returns bf16, the precision the MMA consumes.
__device__ __forceinline__ uint32_t elu1_bf16x2(uint32_t x)
{
    const uint32_t zero = 0u;
    const uint32_t l2e_hi = 0x3FB93FB9u;   // bf16(1.4453125) in both halves
    const uint32_t l2e_lo = 0xBB2CBB2Cu;   // bf16(log2 e - 1.4453125) = -0.00262451 in both halves
    uint32_t neg, pos, t, arg, ex, r;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(neg) : "r"(x), "r"(zero));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(pos) : "r"(x), "r"(zero));
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(t) : "r"(neg), "r"(l2e_lo));
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(arg) : "r"(neg), "r"(l2e_hi), "r"(t));
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

// Symmetric second-order Taylor feature f (0 <= f < 192) of x[16]:
// [1 | x_a/c1 | x_a^2/c2 | sqrt2 x_a x_b / c2 (a < b, row-major) | 0...].
template <int D>
__device__ __forceinline__ float taylor_sym_feature(const float *x, int f, float inv_c1, float inv_c2,
                                                    float r2_inv_c2)
{
    if (f == 0) return 1.f;
    if (f <= D) return x[f - 1] * inv_c1;
    if (f <= 2 * D) return x[f - 1 - D] * x[f - 1 - D] * inv_c2;
    int p = f - 1 - 2 * D;
#pragma unroll
    for (int a = 0; a < D - 1; ++a) {
        const int cnt = D - 1 - a;
        if (p < cnt) return x[a] * x[a + 1 + p] * r2_inv_c2;
        p -= cnt;
    }
    return 0.f;
}

// Row index in the 273-feature (full outer product) layout of symmetric
// feature f, and its second position (or -1) and scale.
template <int D>
__device__ __forceinline__ void taylor_sym_to_full(int f, int &r1, int &r2, float &scale)
{
    r2 = -1;
    scale = 1.f;
    if (f <= D) { r1 = f; return; }
    if (f <= 2 * D) { const int a = f - 1 - D; r1 = 1 + D + a * D + a; return; }
    int p = f - 1 - 2 * D;
    for (int a = 0; a < D - 1; ++a) {
        const int cnt = D - 1 - a;
        if (p < cnt) {
            const int b = a + 1 + p;
            r1 = 1 + D + a * D + b;
            r2 = 1 + D + b * D + a;
            scale = 0.70710678118654752440f;  // the packed feature carries sqrt(2)
            return;
        }
        p -= cnt;
    }
    r1 = -1;
}

}  // namespace fwd_detail

// MODE 0: full forward (o, den, final state).  MODE 1: state increments of
// each segment only (written to p.ws).  GATED: the gated form (p.logdecay);
// a template flag, so the ungated kernels carry none of its work.
template <class Cfg, int MODE, bool GATED>
__global__ void __launch_bounds__(288, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, const FwdParams p)
{
    using namespace sm100;
    using namespace fwd_detail;
    constexpr int C = Cfg::C, DV = Cfg::DV, NA = Cfg::NA, DQK = Cfg::DQK, FP = Cfg::FP;
    // The d = 128 segment pass reads only K and V, so it takes a second K/V
    // stage in the regions the main pass uses for Q and for P (and the state
    // snapshot), which it leaves unused.
    constexpr bool SEG2 = MODE == 1 && DQK == 128;
    constexpr int STAGES = SEG2 ? 2 : Cfg::STAGES;
    static_assert(!SEG2 || (Cfg::STAGES == 1 && Cfg::OFF_Q + Cfg::QK_TILE <= Cfg::OFF_K &&
                            Cfg::OFF_P % 1024 == 0 && Cfg::OFF_P + Cfg::V_TILE <= Cfg::OFF_BAR),
                  "second segment-pass stage");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    auto stage_k = [&](int s) { return (SEG2 && s == 1) ? smem + Cfg::OFF_Q : smem + Cfg::OFF_K + s * Cfg::QK_TILE; };
    auto stage_v = [&](int s) { return (SEG2 && s == 1) ? smem + Cfg::OFF_P : smem + Cfg::OFF_V + s * Cfg::V_TILE; };
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *mma_bar = tma_bar + 2;
    uint64_t *x_bar = tma_bar + 5;   // MODE 0: the scores (MMA1) alone, so the mask need not wait for MMA3
    uint64_t *k_bar = tma_bar + 6;   // MODE 0, d = 128, ungated: MMA1 and MMA3 done with the K tile
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_bar + 3);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tma_bar + 4);

    // 288 threads.  Workers 0..255: warp w reaches TMEM lanes 32 (w % 4) .. + 31
    // and takes column half w / 4 of the row it owns there.  Warp 8: its first
    // thread issues the MMAs and refills the load stages, so that no worker
    // stalls behind the tensor pipe's issue queue; every thread meets at the
    // block barriers.
    // Launched as a programmatic dependent: nothing in global memory is read
    // or written before the previous kernel of the stream has completed; the
    // next one may then take the SMs this grid leaves.
    sm100::grid_dependency_wait();
    sm100::launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, half = warp >> 2, row = wq * 32 + lane;
    const bool worker = tid < 256, issuer = tid == 256;
    const int bh = blockIdx.x / p.P, seg = blockIdx.x % p.P;   // bh: the state slice
    // This slice's tokens: fixed length N at rows bh*N.. of a [BH, N, *] tensor
    // (TMA coordinates (x, t, bh)), or packed sequence n at rows h*T + cu[n]..
    // of a [H, T, *] tensor (TMA coordinates (x, cu[n] + t, h)).
    int N = p.N, nchunks = p.nchunks, nseg = p.P, tz = bh, t_base = 0;
    long long row0 = (long long)bh * p.N;
    if (p.cu) {
        const int n = bh / p.H, h = bh - n * p.H;
        const int a = p.cu[n], b = p.cu[n + 1];
        if (a < 0 || b < a || b > p.T || b - a > p.max_len) {
            if (tid == 0 && seg == 0) report(kStatusCheck);
            return;
        }
        N = b - a;
        nchunks = (N + C - 1) / C;
        nseg = max(1, (nchunks + p.cps - 1) / p.cps);
        if (seg >= nseg) return;   // a shorter sequence: no chunks for this segment
        tz = h;
        t_base = a;
        row0 = (long long)h * p.T + a;
    }
    if (MODE == 1 && seg == nseg - 1) return;  // the last segment's increment is never read
    const int c_begin = seg * p.cps;
    const int c_end = min(nchunks, c_begin + p.cps);

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) mbar_init(&tma_bar[s], 1);
        mbar_init(mma_bar, 1);
        mbar_init(x_bar, 1);
        mbar_init(k_bar, 1);
        *abort_flag = 0;
        mbar_init_fence();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        if (MODE == 0) prefetch_tensormap(&tm_o);
    }
    if (warp == 0) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    // Constant normaliser block of every V stage: column DV of V_aug = 1.
    for (int s = 0; s < STAGES && tid < C; ++s) {
        uint8_t *blk = stage_v(s) + (DV / 16) * Cfg::V_BLK;
        const int r = tid;  // C == 128 rows
        uint4 *row = reinterpret_cast<uint4 *>(blk + (r >> 3) * 256 + (r & 7) * 32);
        const int one_chunk = 0 ^ ((r >> 2) & 1);
        row[one_chunk] = make_uint4(pack_bf16(1.f, 0.f), 0u, 0u, 0u);
        row[one_chunk ^ 1] = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;

    auto issue_tma = [&](int chunk, int s) {
        const int t0 = chunk * C;
        mbar_arrive_expect_tx(&tma_bar[s], MODE == 0 ? Cfg::TX_BYTES : Cfg::TX_BYTES - C * DQK * 2);
        uint8_t *q_dst = smem + Cfg::OFF_Q + s * Cfg::QK_TILE;
        uint8_t *k_dst = stage_k(s);
        constexpr int QBOX = Cfg::TAYLOR ? 16 : 64;
        for (int x = 0; x < DQK; x += QBOX) {
            const int off = Cfg::TAYLOR ? 0 : (x / 64) * C * 128;
            if (MODE == 0) tma_load_3d(q_dst + off, &tm_q, &tma_bar[s], x, t_base + t0, tz);
            tma_load_3d(k_dst + off, &tm_k, &tma_bar[s], x, t_base + t0, tz);
        }
        uint8_t *v_dst = stage_v(s);
        for (int x = 0; x < DV; x += 16)
            tma_load_3d(v_dst + (x / 16) * Cfg::V_BLK, &tm_v, &tma_bar[s], x, t_base + t0, tz);
    };
    // The d = 128 full forward (one stage, ungated) loads a chunk's K as soon as
    // MMA1 and MMA3 have finished with the previous chunk's phi(K), and its Q
    // and V once MMA2 has completed: the K bytes are added to the phase ahead
    // of the arrival that the Q and V copies bring.
    constexpr bool EARLYK128 = MODE == 0 && DQK == 128 && !GATED && STAGES == 1;
    auto issue_k = [&](int chunk, int s) {
        mbar_expect_tx(&tma_bar[s], C * DQK * 2);
        for (int x = 0; x < DQK; x += 64)
            tma_load_3d(stage_k(s) + (x / 64) * C * 128, &tm_k, &tma_bar[s], x, t_base + chunk * C, tz);
    };
    auto issue_qv = [&](int chunk, int s) {
        const int t0 = chunk * C;
        mbar_arrive_expect_tx(&tma_bar[s], Cfg::TX_BYTES - C * DQK * 2);
        for (int x = 0; x < DQK; x += 64)
            tma_load_3d(smem + Cfg::OFF_Q + s * Cfg::QK_TILE + (x / 64) * C * 128, &tm_q, &tma_bar[s], x, t_base + t0, tz);
        for (int x = 0; x < DV; x += 16)
            tma_load_3d(stage_v(s) + (x / 16) * Cfg::V_BLK, &tm_v, &tma_bar[s], x, t_base + t0, tz);
    };
    uint32_t k_phase = 0;

    bool have_state = false;
    constexpr bool gated = GATED;
    // gated form: per-segment sums of the log gates follow the increments in
    // the workspace, [slices, P]
    float *ws_log = p.ws ? p.ws + (size_t)(gridDim.x / p.P) * p.P * FP * NA : nullptr;
    float lsum_before = 0.f;   // gated: sum of the gates of the earlier segments
    if (MODE == 0 && gated)
        for (int s2 = 0; s2 < seg; ++s2) lsum_before += ws_log[(size_t)bh * p.P + s2];
    // ---- starting state of this segment: the state entering the sequence (if
    // given) plus the sum of the earlier segments' increments; gated, each
    // earlier term first decays by the gates of the segments after it:
    // acc <- exp(L_seg) acc + dS_seg, from the entering state through seg - 1
    if (MODE == 0 && (seg > 0 || p.s_in)) {
        for (int t = 0; t < (worker ? Cfg::NT : 0); ++t) {
            const int m = Cfg::tile_m(t);
            const int r = (m == 128) ? row : ((lane < 16) ? wq * 16 + lane : -1);
            const int f = r < 0 ? -1 : Cfg::tile_f0(t) + r;
            for (int c0 = 16 * half; c0 < NA; c0 += 32) {
                float acc[16], sin16[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[e] = sin16[e] = 0.f;
                if (f >= 0 && f < FP) {
                    if (p.s_in && f < Cfg::FSYM) {
                        // boundary rows of internal row f (Taylor: the symmetric pair, scaled)
                        const int F = !Cfg::TAYLOR ? DQK : p.sym_state ? Cfg::FSYM : 1 + DQK + DQK * DQK;
                        int r1 = f, r2 = -1;
                        float sc = 1.f;
                        if (Cfg::TAYLOR && !p.sym_state) taylor_sym_to_full<16>(f, r1, r2, sc);
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int col = c0 + e;
                            float x = 0.f;
                            if (col < DV) {
                                x = p.s_in[((size_t)bh * F + r1) * DV + col];
                                if (r2 >= 0) x += p.s_in[((size_t)bh * F + r2) * DV + col];
                            } else if (col == DV) {
                                x = p.z_in[(size_t)bh * F + r1];
                                if (r2 >= 0) x += p.z_in[(size_t)bh * F + r2];
                            }
                            sin16[e] = sc * x;
                        }
                    }
                    if (gated) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) acc[e] = sin16[e];
                        for (int s2 = 0; s2 < seg; ++s2) {
                            const float d = __expf(ws_log[(size_t)bh * p.P + s2]);
                            const float *src = p.ws + ((size_t)(bh * p.P + s2) * FP + f) * NA + c0;
#pragma unroll
                            for (int e = 0; e < 16; ++e) acc[e] = fmaf(acc[e], d, src[e]);
                        }
                    } else {
                        for (int s2 = 0; s2 < seg; ++s2) {
                            const float *src = p.ws + ((size_t)(bh * p.P + s2) * FP + f) * NA + c0;
#pragma unroll
                            for (int e = 0; e < 16; ++e) acc[e] += src[e];
                        }
#pragma unroll
                        for (int e = 0; e < 16; ++e) acc[e] += sin16[e];
                    }
                }
                tmem_st16(tmem + lane_base + Cfg::COL_S + t * NA + c0, acc);
                if (f >= 0 && f < FP) {
                    uint8_t *sS = smem + Cfg::OFF_S;
#pragma unroll
                    for (int e = 0; e < 16; e += 8) {
                        uint4 u = make_uint4(pack_bf16(acc[e], acc[e + 1]), pack_bf16(acc[e + 2], acc[e + 3]),
                                             pack_bf16(acc[e + 4], acc[e + 5]), pack_bf16(acc[e + 6], acc[e + 7]));
                        *reinterpret_cast<uint4 *>(sS + sw32_off(f, c0 + e, FP)) = u;
                    }
                }
            }
        }
        tmem_st_wait();
        have_state = true;
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (tid == 0)
        for (int s = 0; s < STAGES && c_begin + s < c_end; ++s) issue_tma(c_begin + s, s);

    uint32_t mma_phase = 0, x_phase = 0;
    const float inv_c1 = p.inv_c1, inv_c2 = p.inv_c2, r2_inv_c2 = p.inv_c2 * 1.41421356237309504880f;
    float seg_log = 0.f;   // gated: sum of this segment's gates so far
    float *gL = reinterpret_cast<float *>(smem + Cfg::OFF_G);   // [C] prefix sums of the chunk's gates
    float *gTot = gL + C;                                         // [4] per-warp totals

    // Gated form, elu: multiply this thread's half of row `row` of a phi tile by rs.
    auto scale_row_half = [&](uint8_t *tile, float rs) {
#pragma unroll
        for (int col = half * (DQK / 2); col < (half + 1) * (DQK / 2); col += 8) {
            const uint32_t a = smem_addr(tile + sw128_off(row, col));
            float x8[8];
            unpack8(lds128(a), x8);
            sts128(a, make_uint4(pack_bf16(rs * x8[0], rs * x8[1]), pack_bf16(rs * x8[2], rs * x8[3]),
                                 pack_bf16(rs * x8[4], rs * x8[5]), pack_bf16(rs * x8[6], rs * x8[7])));
        }
    };
    // Gated form: S_aug in TMEM <- exp(l) S_aug (this thread's lanes and columns).
    auto decay_state = [&](float l) {
        const float dl = __expf(l);
#pragma unroll 1
        for (int t = 0; t < Cfg::NT; ++t) {
#pragma unroll 1
            for (int c0 = 16 * half; c0 < NA; c0 += 32) {
                float v[16];
                tmem_ld16(tmem + lane_base + Cfg::COL_S + t * NA + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] *= dl;
                tmem_st16(tmem + lane_base + Cfg::COL_S + t * NA + c0, v);
            }
        }
        tmem_st_wait();
    };

    // MMA3: S_aug (+)= phi(K_c)^T V_aug, issued by one thread.
    auto issue_state_mma = [&](uint32_t aK, uint32_t aV, bool acc0) {
#pragma unroll
        for (int t = 0; t < Cfg::NT; ++t) {
            const int m = Cfg::tile_m(t);
            const uint32_t idesc = idesc_bf16(m, NA, 1, 1);
            const uint32_t a_base = aK + (Cfg::tile_f0(t) / 64) * (C * 128);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                mma_bf16(tmem + Cfg::COL_S + t * NA,
                         smem_desc(a_base + kk * 2048, C * 128, 1024, kSw128),
                         smem_desc(aV + kk * 512, Cfg::V_BLK, 256, kSw32), idesc, acc0 || kk > 0);
            }
        }
    };

    // Taylor, full forward: phi(Q) goes to TMEM (columns COL_PQ + 40 h for the
    // row's half h: K-step kk of MMA2's state term takes columns 8 kk .. 8 kk + 7);
    // ungated, the next chunk's phi(K) is built into the other phi(K) tile while
    // this chunk's MMA2 runs.
    constexpr bool EARLYK = Cfg::TAYLOR && MODE == 0 && !GATED;
    // elu with two load stages, full forward: the next chunk's phi(Q) and phi(K)
    // are formed in place in its stage (already landed) while this chunk's MMA2
    // runs (the gated form scales them after MMA1, as before)
    constexpr bool EARLYPHI = !Cfg::TAYLOR && MODE == 0 && STAGES == 2;
    // elu(x)+1 in place on this thread's half of row `row` of Q and K (K rows
    // past `kvalid_rows` zeroed)
    auto elu_phi_in_place = [&](uint8_t *tq, uint8_t *tk, int kvalid_rows, bool do_q) {
#pragma unroll 1
        for (int m = do_q ? 0 : 1; m < 2; ++m) {
            uint8_t *tile = m == 0 ? tq : tk;
            const bool zero = m == 1 && row >= kvalid_rows;
#pragma unroll
            for (int col = half * (DQK / 2); col < (half + 1) * (DQK / 2); col += 8) {
                const uint32_t a = smem_addr(tile + sw128_off(row, col));
                const uint4 r = lds128(a);
                sts128(a, zero ? make_uint4(0u, 0u, 0u, 0u)
                               : make_uint4(elu1_bf16x2(r.x), elu1_bf16x2(r.y), elu1_bf16x2(r.z), elu1_bf16x2(r.w)));
            }
        }
    };
    auto phi_k_tile = [&](int itk) {   // the phi(K) tile of the range's chunk itk
        return smem + ((EARLYK && (itk & 1)) ? Cfg::OFF_PQ : Cfg::OFF_PK);
    };
    // this thread's half of phi(x) (times rs) for row `row` into an SW128 phi tile
    auto taylor_tile_half = [&](uint8_t *dst, const float *x, bool zero, float rs) {
        auto features = [&](auto h) {
            constexpr int F0 = decltype(h)::value * (Cfg::FT / 2);
#pragma unroll
            for (int f0 = F0; f0 < F0 + Cfg::FT / 2; f0 += 8) {
                float v8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    v8[e] = zero ? 0.f : rs * taylor_sym_feature<16>(x, f0 + e, inv_c1, inv_c2, r2_inv_c2);
                *reinterpret_cast<uint4 *>(dst + sw128_off(row, f0)) =
                    make_uint4(pack_bf16(v8[0], v8[1]), pack_bf16(v8[2], v8[3]), pack_bf16(v8[4], v8[5]),
                               pack_bf16(v8[6], v8[7]));
            }
        };
        if (half == 0) features(std::integral_constant<int, 0>{});
        else features(std::integral_constant<int, 1>{});
    };
    auto taylor_q_tmem = [&](const float *x, float rs) {
        uint32_t w[40];
        auto features = [&](auto h) {
            constexpr int F0 = decltype(h)::value * 80;
#pragma unroll
            for (int e = 0; e < 80; e += 2)
                w[e / 2] = pack_bf16(rs * taylor_sym_feature<16>(x, F0 + e, inv_c1, inv_c2, r2_inv_c2),
                                     rs * taylor_sym_feature<16>(x, F0 + e + 1, inv_c1, inv_c2, r2_inv_c2));
        };
        if (half == 0) features(std::integral_constant<int, 0>{});
        else features(std::integral_constant<int, 1>{});
        tmem_st32(tmem + lane_base + Cfg::COL_PQ + 40 * half, w);
        tmem_st8(tmem + lane_base + Cfg::COL_PQ + 40 * half + 32, w + 32);
        tmem_st_wait();
    };

    for (int chunk = c_begin; chunk < c_end; ++chunk) {
        const int it = chunk - c_begin;
        const int s = it % STAGES;
        const uint32_t tphase = (uint32_t)(it / STAGES) & 1u;
        const int t0 = chunk * C;
        const int nvalid = min(C, N - t0);
        // ---- gated form: L_i = g_{t0} + ... + g_{t0+i} over the chunk (rows past
        // the end add 0), e_i = exp(L_i) scales phi(q_i) for the carried state,
        // w_i = exp(L_last - L_i) scales phi(k_i) for the state update.
        float gate_e = 1.f, gate_w = 1.f, gate_last = 0.f, gate_L = 0.f;
        if (gated) {
            // gates below e^-80 count as e^-80: zero next to any surviving term
            // in fp32, and it keeps L finite, so differences of L never meet inf - inf
            float x = worker && row < nvalid ? fmaxf(p.logdecay[row0 + t0 + row], -80.f) : 0.f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            if (worker && half == 0 && lane == 31) gTot[wq] = x;
            __syncthreads();
            float before = 0.f;
#pragma unroll
            for (int w2 = 0; w2 < 4; ++w2) {
                if (w2 < wq) before += gTot[w2];
                gate_last += gTot[w2];
            }
            gate_L = x + before;
            if (half == 0) gL[row] = gate_L;
            gate_e = __expf(gate_L);
            gate_w = __expf(gate_last - gate_L);
            seg_log += gate_last;
        }
        // (the issuer waits too: its MMAs read the stage)
        if (!mbar_wait(&tma_bar[s], tphase)) *abort_flag = 1;
        uint8_t *sQ = smem + Cfg::OFF_Q + s * Cfg::QK_TILE;
        uint8_t *sK = stage_k(s);
        uint8_t *sV = stage_v(s);
        uint8_t *sPQ = sQ;   // elu: phi in place (Taylor: phi(Q) in TMEM)
        uint8_t *sPK = Cfg::TAYLOR ? phi_k_tile(it) : sK;

        // ---- feature maps (token row `row`, column half `half`)
        if (worker) {
            const int i = row;
            const bool kvalid = i < nvalid;
            if (!Cfg::TAYLOR) {
                // EARLYPHI: chunks after the first were converted during the previous one
                if (!(EARLYPHI && it > 0)) elu_phi_in_place(sQ, sK, nvalid, MODE == 0);
                // segment pass, gated: phi(K) feeds only MMA3 here, scale it now
                if (MODE == 1 && gated) scale_row_half(sK, gate_w);
            } else {
                float x[16];
                if (MODE == 0) {
                    unpack8(*reinterpret_cast<const uint4 *>(sQ + sw32_off(i, 0, C)), x);
                    unpack8(*reinterpret_cast<const uint4 *>(sQ + sw32_off(i, 8, C)), x + 8);
                    taylor_q_tmem(x, gate_e);   // gate_e = 1 ungated
                }
                if (!(EARLYK && it > 0)) {   // EARLYK: built during the previous chunk
                    unpack8(*reinterpret_cast<const uint4 *>(sK + sw32_off(i, 0, C)), x);
                    unpack8(*reinterpret_cast<const uint4 *>(sK + sw32_off(i, 8, C)), x + 8);
                    taylor_tile_half(sPK, x, !kvalid, gate_w);
                }
            }
        }
        // segment pass, gated: the carried state decays before MMA3 adds to it
        if (worker && MODE == 1 && gated && have_state) decay_state(gate_last);
        // the previous chunk's y store has read its staging tile (the P tile,
        // which the mask below writes again)
        if (MODE == 0 && issuer && it > 0) bulk_wait_read();
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (*abort_flag) break;

        // ---- MMA1 (scores) and MMA3 (state update)
        if (issuer) {
            const uint32_t aQ = smem_addr(sPQ), aK = smem_addr(sPK), aV = smem_addr(sV);
            if (MODE == 0) {
                if (Cfg::TAYLOR) {
                    const uint32_t qa = smem_addr(sQ), ka = smem_addr(sK);
                    mma_bf16(tmem + Cfg::COL_O, smem_desc(qa, 16, 256, kSw32), smem_desc(ka, 16, 256, kSw32),
                             idesc_bf16(128, 128, 0, 0), false);
                } else {
#pragma unroll
                    for (int kk = 0; kk < DQK / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * (C * 128) + (kk & 3) * 32;
                        mma_bf16(tmem + Cfg::COL_O, smem_desc(aQ + off, 16, 1024, kSw128),
                                 smem_desc(aK + off, 16, 1024, kSw128), idesc_bf16(128, 128, 0, 0), kk > 0);
                    }
                }
            }
            if (MODE == 0) mma_commit(x_bar);
            // MMA3 runs under the mask step; the commit after MMA2 covers it
            if (!gated || MODE == 1) issue_state_mma(aK, aV, have_state);
            if (EARLYK128) mma_commit(k_bar);
            if (MODE == 1) mma_commit(mma_bar);
        }
        if (MODE == 0) {
            if (worker && !mbar_wait(x_bar, x_phase)) *abort_flag = 1;
            x_phase ^= 1u;
        } else {
            if (!mbar_wait(mma_bar, mma_phase)) *abort_flag = 1;
            mma_phase ^= 1u;
        }
        tc_fence_after();
        if (!gated || MODE == 1) have_state = true;

        if (MODE == 1) {
            __syncthreads();
            if (issuer && it + STAGES < c_end - c_begin) issue_tma(chunk + STAGES, s);
            if (*abort_flag) break;
            continue;
        }

        // ---- causal mask -> P (bf16, K-major SW128); keys of this thread's half
        if (worker) {
            const int i = row;
            uint8_t *sP = smem + Cfg::OFF_P;
#pragma unroll 1
            for (int j0 = half * (C / 2); j0 < (half + 1) * (C / 2); j0 += 32) {
                float a[32];
                tmem_ld32(tmem + lane_base + Cfg::COL_O + j0, a);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int j = j0 + e;
                    float w = a[e];
                    if (Cfg::TAYLOR) w = 1.f + w * p.k1 + w * w * p.k2;
                    if (gated) w *= __expf(gate_L - gL[j]);   // a_{j+1} ... a_i
                    a[e] = (j <= i) ? w : 0.f;
                }
#pragma unroll
                for (int e = 0; e < 32; e += 8)
                    *reinterpret_cast<uint4 *>(sP + sw128_off(i, j0 + e)) =
                        make_uint4(pack_bf16(a[e], a[e + 1]), pack_bf16(a[e + 2], a[e + 3]),
                                   pack_bf16(a[e + 4], a[e + 5]), pack_bf16(a[e + 6], a[e + 7]));
            }
        }
        if (gated && worker) {
            // elu: phi tiles are also MMA1's operands, so they are scaled only
            // now that MMA1 has completed (Taylor scaled them when computing them)
            if (!Cfg::TAYLOR) {
                scale_row_half(sPQ, gate_e);
                scale_row_half(sPK, gate_w);
            }
            // the carried state decays by the chunk's whole gate before MMA3 adds to it
            if (have_state) decay_state(gate_last);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---- MMA2: O_aug = P V_aug + phi(Q) S_snap
        if (issuer) {
            const uint32_t aP = smem_addr(smem + Cfg::OFF_P), aV = smem_addr(sV);
            const uint32_t idesc = idesc_bf16(128, NA, 0, 1);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                const uint32_t off = (kk >> 2) * (C * 128) + (kk & 3) * 32;
                mma_bf16(tmem + Cfg::COL_O, smem_desc(aP + off, 16, 1024, kSw128),
                         smem_desc(aV + kk * 512, Cfg::V_BLK, 256, kSw32), idesc, kk > 0);
            }
            if (chunk > 0 || p.s_in) {
                const uint32_t aQ = smem_addr(sPQ), aS = smem_addr(smem + Cfg::OFF_S);
#pragma unroll
                for (int kk = 0; kk < FP / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (C * 128) + (kk & 3) * 32;
                    if constexpr (Cfg::TAYLOR)
                        mma_bf16_ts(tmem + Cfg::COL_O, tmem + Cfg::COL_PQ + kk * 8,
                                    smem_desc(aS + kk * 512, Cfg::S_BLK, 256, kSw32), idesc, true);
                    else
                        mma_bf16(tmem + Cfg::COL_O, smem_desc(aQ + off, 16, 1024, kSw128),
                                 smem_desc(aS + kk * 512, Cfg::S_BLK, 256, kSw32), idesc, true);
                }
            }
            if (gated) issue_state_mma(smem_addr(sPK), aV, have_state);
            mma_commit(mma_bar);
            if (EARLYK128 && it + 1 < c_end - c_begin) {
                if (!mbar_wait(k_bar, k_phase)) *abort_flag = 1;
                k_phase ^= 1u;
                issue_k(chunk + 1, s);
            }
        }
        if (EARLYPHI && worker && chunk + 1 < c_end) {
            const int s1 = (it + 1) % STAGES;
            if (!mbar_wait(&tma_bar[s1], (uint32_t)((it + 1) / STAGES) & 1u)) *abort_flag = 1;
            elu_phi_in_place(smem + Cfg::OFF_Q + s1 * Cfg::QK_TILE, smem + Cfg::OFF_K + s1 * Cfg::QK_TILE,
                             min(C, N - t0 - C), true);
        }
        if (EARLYK && worker && chunk + 1 < c_end) {
            // the next chunk's phi(K) into the other tile (MMA3 two chunks back
            // read it last and has finished) while MMA2 runs
            const int s1 = (it + 1) % STAGES;
            if (!mbar_wait(&tma_bar[s1], (uint32_t)((it + 1) / STAGES) & 1u)) *abort_flag = 1;
            const uint8_t *sK1 = smem + Cfg::OFF_K + s1 * Cfg::QK_TILE;
            float x[16];
            unpack8(*reinterpret_cast<const uint4 *>(sK1 + sw32_off(row, 0, C)), x);
            unpack8(*reinterpret_cast<const uint4 *>(sK1 + sw32_off(row, 8, C)), x + 8);
            taylor_tile_half(phi_k_tile(it + 1), x, row >= min(C, N - t0 - C), 1.f);
        }
        if (!mbar_wait(mma_bar, mma_phase)) *abort_flag = 1;
        mma_phase ^= 1u;
        tc_fence_after();
        if (gated) have_state = true;
        if (issuer && it + STAGES < c_end - c_begin) {
            if (EARLYK128) issue_qv(chunk + STAGES, s);
            else issue_tma(chunk + STAGES, s);
        }

        // ---- outputs: y = num / den (this thread's half of the value columns).
        // y goes to the P tile (free once MMA2 has completed) as SW128 rows and
        // leaves by one TMA store after the chunk's last barrier: at fixed
        // length rows past the slice's end are clipped by the tensor map; a
        // packed sequence's partial last chunk would reach into the next
        // sequence's rows, so there the rows of this sequence are stored directly.
        const bool tma_y = !p.cu || nvalid == C;
        if (worker) {
            const int i = row;
            constexpr int DH = DV / 2;
            float o[DH], d16[16];
            tmem_ld16(tmem + lane_base + Cfg::COL_O + DV, d16);   // den in column DV
#pragma unroll
            for (int c0 = 0; c0 < DH; c0 += 16) tmem_ld16(tmem + lane_base + Cfg::COL_O + half * DH + c0, o + c0);
            tmem_ld_wait();
            const float den = d16[0];
            const float inv = 1.f / den;
            if (tma_y) {
                uint8_t *sY = smem + Cfg::OFF_P;
#pragma unroll
                for (int c0 = 0; c0 < DH; c0 += 8) {
                    const int col = half * DH + c0;
                    *reinterpret_cast<uint4 *>(sY + (col / 64) * (C * 128) + sw128_off(i, col % 64)) =
                        make_uint4(pack_bf16(o[c0] * inv, o[c0 + 1] * inv), pack_bf16(o[c0 + 2] * inv, o[c0 + 3] * inv),
                                   pack_bf16(o[c0 + 4] * inv, o[c0 + 5] * inv), pack_bf16(o[c0 + 6] * inv, o[c0 + 7] * inv));
                }
            } else if (i < nvalid) {
                __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) + (size_t)(row0 + t0 + i) * DV + half * DH;
#pragma unroll
                for (int c0 = 0; c0 < DH; c0 += 8)
                    *reinterpret_cast<uint4 *>(orow + c0) =
                        make_uint4(pack_bf16(o[c0] * inv, o[c0 + 1] * inv), pack_bf16(o[c0 + 2] * inv, o[c0 + 3] * inv),
                                   pack_bf16(o[c0 + 4] * inv, o[c0 + 5] * inv), pack_bf16(o[c0 + 6] * inv, o[c0 + 7] * inv));
            }
            if (p.den_out && half == 0 && i < nvalid) p.den_out[row0 + t0 + i] = den;
        }
        // ---- state snapshot for the next chunk (bf16, MN-major SW32)
        if (worker && chunk + 1 < c_end) {
            uint8_t *sS = smem + Cfg::OFF_S;
#pragma unroll
            for (int t = 0; t < Cfg::NT; ++t) {
                const int m = Cfg::tile_m(t);
                const int r = (m == 128) ? row : ((lane < 16) ? wq * 16 + lane : -1);
                const int f = r < 0 ? -1 : Cfg::tile_f0(t) + r;
#pragma unroll
                for (int c0 = 16 * half; c0 < NA; c0 += 32) {
                    float v[16];
                    tmem_ld16(tmem + lane_base + Cfg::COL_S + t * NA + c0, v);
                    tmem_ld_wait();
                    if (f >= 0 && f < FP) {
                        *reinterpret_cast<uint4 *>(sS + sw32_off(f, c0, FP)) =
                            make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                                       pack_bf16(v[6], v[7]));
                        *reinterpret_cast<uint4 *>(sS + sw32_off(f, c0 + 8, FP)) =
                            make_uint4(pack_bf16(v[8], v[9]), pack_bf16(v[10], v[11]), pack_bf16(v[12], v[13]),
                                       pack_bf16(v[14], v[15]));
                    }
                }
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (MODE == 0 && issuer && tma_y && !*abort_flag) {
            for (int x = 0; x < DV; x += 64)
                tma_store_3d(&tm_o, smem + Cfg::OFF_P + (x / 64) * (C * 128), x, t_base + t0, tz);
            bulk_commit();
        }
        if (*abort_flag) break;
    }
    // the last y stores have completed (their staging tile and the block's
    // shared memory outlive them)
    if (MODE == 0 && issuer) bulk_wait_all();

    // ---- segment increment (MODE 1) or final state (MODE 0, last segment)
    const bool write_ws = (MODE == 1);
    const bool write_final = (MODE == 0) && (seg == nseg - 1) && (p.s_out || p.z_out) && !*abort_flag;
    if (write_ws && gated && tid == 0 && !*abort_flag) ws_log[(size_t)bh * p.P + seg] = seg_log;
    // gated: the entering state's antisymmetric part (restored below) has
    // decayed by every gate of the sequence
    const float skew_decay = gated ? __expf(lsum_before + seg_log) : 1.f;
    if (worker && (write_ws || write_final) && !*abort_flag) {
#pragma unroll 1
        for (int t = 0; t < Cfg::NT; ++t) {
            const int m = Cfg::tile_m(t);
            const int r = (m == 128) ? row : ((lane < 16) ? wq * 16 + lane : -1);
            const int f = r < 0 ? -1 : Cfg::tile_f0(t) + r;
#pragma unroll 1
            for (int c0 = 16 * half; c0 < NA; c0 += 32) {
                float v[16];
                tmem_ld16(tmem + lane_base + Cfg::COL_S + t * NA + c0, v);
                tmem_ld_wait();
                if (!have_state) {   // an empty packed sequence with no entering state
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = 0.f;
                }
                if (f < 0 || f >= FP) continue;
                if (write_ws) {
                    float *dst = p.ws + ((size_t)(bh * p.P + seg) * FP + f) * NA + c0;
#pragma unroll
                    for (int e = 0; e < 16; ++e) dst[e] = v[e];
                    continue;
                }
                if (f >= Cfg::FSYM) continue;
                const int F = !Cfg::TAYLOR ? DQK : p.sym_state ? Cfg::FSYM : 1 + DQK + DQK * DQK;
                int r1, r2;
                float sc;
                if (Cfg::TAYLOR && !p.sym_state) {
                    taylor_sym_to_full<16>(f, r1, r2, sc);
                } else {
                    r1 = f; r2 = -1; sc = 1.f;
                }
                for (int e = 0; e < 16; ++e) {
                    const int col = c0 + e;
                    const float val = v[e] * sc;
                    // a packed row holds the symmetric part of a given entering state;
                    // its antisymmetric part (zero for any state a prefill produces) is
                    // added back so the returned state is exact
                    float skew = 0.f;
                    if (r2 >= 0 && p.s_in)
                        skew = 0.5f * skew_decay * (col < DV ? p.s_in[((size_t)bh * F + r1) * DV + col] -
                                                      p.s_in[((size_t)bh * F + r2) * DV + col]
                                                : (col == DV ? p.z_in[(size_t)bh * F + r1] - p.z_in[(size_t)bh * F + r2]
                                                             : 0.f));
                    if (col < DV) {
                        if (p.s_out) {
                            p.s_out[((size_t)bh * F + r1) * DV + col] = val + skew;
                            if (r2 >= 0) p.s_out[((size_t)bh * F + r2) * DV + col] = val - skew;
                        }
                    } else if (col == DV && p.z_out) {
                        p.z_out[(size_t)bh * F + r1] = val + skew;
                        if (r2 >= 0) p.z_out[(size_t)bh * F + r2] = val - skew;
                    }
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
