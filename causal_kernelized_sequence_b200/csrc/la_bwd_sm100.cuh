// la_bwd_sm100.cuh -- tensor-core backward of causal linear attention (bf16
// I/O), tcgen05 + TMA, for three shapes: the elu(x)+1 map with
// d_qk = d_v = 128 or 64, and the BASED second-order Taylor map with d' = 16
// and d_v = 64 (both the full and the folded map: their phi(q).phi(k) and so
// their gradients are the same).
//
// The pages give no backward pass; this is the derivative of the BASED page's
// Knowl 3 parallel form, computed chunk by chunk (128 tokens) with the same
// augmented-value trick as the forward: V_aug = [V | 1 | 0..], S_aug = [S | z],
// G'_i = [g_i | dden_i | 0..] with g_i = dout_i / den_i, dden_i = -g_i . y_i.
// Then, for a chunk c with state S_aug entering it and R_aug = sum over the
// later chunks of phi(q_i) G'_i^T,
//
//   forward-order pass (dq), in units of den_i per row i:
//     A   = phi(Q) phi(K)^T, P = A masked to j <= i
//     O   = P V_aug + phi(Q) S_aug          -> y, den; G'' = den G' = [dO | -dO.y]
//     dA  = G'' V_aug^T,  dP = dA masked to j <= i
//     dphi(Q) = (dP phi(K) + G'' S_aug^T) / den   -> dq = J_phi(q)^T dphi(q)
//     S_aug += phi(K)^T V_aug
//   reverse-order pass (dk, dv):
//     A^T = phi(K) phi(Q)^T, P^T; dA^T = V_aug G'^T, dP^T (masked to i >= j)
//     dV  = P^T G + phi(K) R                 (R = first d_v columns of R_aug)
//     dphi(K) = dP^T phi(Q) + V_aug R_aug^T  -> dk = J_phi(k)^T dphi(k)
//     R_aug += phi(Q)^T G'
//
// The maps.  elu: J_phi(x)^T is the diagonal elu'(x) = 1 for x > 0 and
// exp(x) = phi(x) otherwise, i.e. min(phi(x), 1).  Taylor: the scores come
// from the raw Q K^T (K = 16) through the closed form
// 1 + s/sqrt(d') + s^2/(2 d') (BASED page, Knowl 3), and phi is the folded
// map's 153 features (padded to 160 with zeros) in a separate shared-memory
// tile; J_phi(x)^T dphi maps the 160 feature derivatives back to the 16
// coordinates on the CUDA cores (linear features 1/d'^(1/4), squares
// 2 x_a / (sqrt2 sqrt d'), pairs x_b / sqrt(d') and x_a / sqrt(d')).
//
// den and dden are recomputed in fp32 in the forward-order pass (so no
// rounded forward output enters the gradient) and kept per token in the
// workspace for the reverse pass.  Sequences are split into the forward's
// segments; the state entering a segment is the sum of bwd_sstate_kernel's
// increments (S) of the earlier segments, and R that of bwd_rstate_kernel's
// increments of the later ones.
//
// dphi(Q) is replaced by its component orthogonal to phi(q_i) before the
// chain rule.  That is exact: y_i is unchanged when phi(q_i) is scaled, so
// dphi(q_i) . phi(q_i) = 0 in exact arithmetic and only rounding noise is
// removed (elu features are all ~1, so that noise is large next to dq).  For
// the Taylor map the projection is applied after the chain rule, with
// |phi(x)|^2 = 1 + |x|^2/sqrt(d') + |x|^4/(2 d') and
// J_phi(x)^T phi(x) = x (1/sqrt(d') + |x|^2/d') in closed form.
// The elu forward-order pass runs its MMAs on fp16 operands (phi - 1 carries
// dq and keeps 3 more bits in fp16); the Taylor map, whose features are not
// clustered near one value, runs on bf16 with a bf16 remainder on the state
// and on G'' for the inter-chunk term.  The reverse pass uses bf16 operands,
// with P^T and G' each split into a bf16 head and a bf16 remainder on the
// products that carry dk.
//
// Token or feature row i <-> TMEM lane i.  The Taylor state (160 feature
// rows) is two TMEM tiles, M = 128 (features 0..127) and M = 64 (features
// 128..191, of which 128..159 are kept: row 128 + 16 q + l in lane 32 q + l,
// l < 16); the elu d = 64 state is one M = 64 tile in the same layout.
// bwd_dq_kernel and bwd_dkdv_kernel run 256 threads: warps w and w + 4 share
// the lanes of one 32-row quadrant and split every per-row step by columns,
// exchanging row reductions through shared memory.  The S and R increment
// passes run 256 threads on three load stages for the elu shapes
// (bwd_sstate3_kernel, bwd_rstate3_kernel: a chunk's MMA runs under the next
// chunk's conversion) and 128 threads, one per row, on two stages for the
// Taylor map (bwd_sstate_kernel, bwd_rstate_kernel).  Each block takes a
// chunk's steps in order; every mbarrier wait is bounded.
#pragma once

#include <type_traits>

#include "la_device.cuh"
#include "la_prefill_sm100.cuh"
#include "sm100.cuh"

namespace la {

template <int D_, int DV_, bool TAYLOR_>
struct BwdCfg {
    static constexpr int D = D_, DV = DV_;
    static constexpr bool TAYLOR = TAYLOR_;
    static constexpr bool F16 = !TAYLOR;                 // fp16 operands in the forward-order pass
    static constexpr int C = 128;
    static constexpr int NA = DV + 16;                   // value columns + normaliser block
    static constexpr int F = TAYLOR ? 160 : D;           // feature rows of the state
    static constexpr int FT = TAYLOR ? 192 : D;          // width of a phi tile (64-feature SW128 blocks)
    static constexpr int NT = TAYLOR ? 2 : 1;            // state tiles in TMEM
    static __host__ __device__ constexpr int tile_m(int t) { return TAYLOR ? (t == 0 ? 128 : 64) : (D == 128 ? 128 : 64); }
    static __host__ __device__ constexpr int tile_f0(int t) { return 128 * t; }
    static constexpr int NA_SPLIT = ((NA / 16 + 1) / 2) * 16;   // a row's first thread takes columns [0, NA_SPLIT)
    // shared memory (bytes; SW128 regions 1024-aligned, SW32 regions 256-aligned)
    static constexpr int PHI_TILE = C * FT * 2;          // phi(Q) or phi(K) (elu: the loaded tile, phi in place)
    static constexpr int RAW = TAYLOR ? C * 32 : 0;      // raw Q or K tile (Taylor, one 16-column SW32 block)
    static constexpr int BLK = C * 32;                   // one 16-column SW32 block of 128 rows
    static constexpr int VG_TILE = (NA / 16) * BLK;      // V_aug or G'
    static constexpr int S_BLK = F * 32;                 // 16 columns of the F x NA state
    static constexpr int S_TILE = (NA / 16) * S_BLK;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + PHI_TILE;
    static constexpr int OFF_V = OFF_K + PHI_TILE;
    static constexpr int OFF_G = OFF_V + VG_TILE;
    static constexpr int OFF_S = OFF_G + VG_TILE;
    // low part of the state (forward-order pass) or of G' (reverse pass)
    static constexpr int SL_TILE = S_TILE > VG_TILE ? S_TILE : VG_TILE;
    static constexpr int OFF_SL = OFF_S + S_TILE;
    static constexpr int OFF_RQ = OFF_SL + SL_TILE;      // raw Q (Taylor)
    static constexpr int OFF_RK = OFF_RQ + RAW;          // raw K (Taylor)
    static constexpr int OFF_BAR = OFF_RK + RAW;
    static constexpr int OFF_RED = OFF_BAR + 128;        // per-row partial sums of the two threads of a row
    static constexpr int RED_FLOATS = 6 * C + (TAYLOR ? 2 * C * 16 : 0);
    // gated form: [C] prefix sums of the gates, [8] quadrant totals, then (reverse
    // pass) [F] the bf16 remainder of R's normaliser column
    static constexpr int OFF_GATE = OFF_RED + RED_FLOATS * 4;
    static constexpr int SMEM_ALLOC = OFF_GATE + (C + 8 + F) * 4 + 1024;
    // TMEM columns.  Forward-order pass: [0, 128) scores -> P | dP; X: O_aug,
    // then dA, then dphi(Q); S: the state tiles; GL: the remainder of G''.
    // Reverse pass: [0, 128) scores -> P^T | dP^T; X: dA^T, then dV, then
    // dphi(K); R: the R_aug tiles; PL: the remainder of dP^T.
    static constexpr int cmax(int a, int b) { return a > b ? a : b; }
    static constexpr int COL_X = C;
    static constexpr int COL_S = COL_X + cmax(cmax(NA, C), F);
    static constexpr int COL_GL = COL_S + NT * NA;
    static constexpr int COL_R = COL_X + cmax(cmax(C, DV), F);
    static constexpr int COL_PL = COL_R + NT * NA;
    static constexpr int TMEM_COLS = 512;
    static_assert(COL_GL + NA / 2 <= 512 && COL_PL + C / 2 <= 512, "TMEM columns");
    static_assert(NT * NA <= 256, "state tiles of the state passes");
    static_assert(PHI_TILE % 1024 == 0 && VG_TILE % 1024 == 0 && S_TILE % 256 == 0 && OFF_RQ % 1024 == 0,
                  "shared-memory alignment");
    static_assert(SL_TILE >= S_TILE && SL_TILE >= VG_TILE && OFF_S + S_TILE >= OFF_G + VG_TILE,
                  "the R snapshot fits the S region and the G' remainder the SL region");
    static_assert(SL_TILE >= C * DV * 2 && OFF_SL % 1024 == 0, "dv staged in the SL region (SW128)");
    static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory");
    // elu state passes (bwd_sstate3_kernel, bwd_rstate3_kernel): three stages of
    // [K or Q tile | V_aug or G'_aug], then barriers and the gate prefix sums
    static constexpr int SP_A = C * D * 2;
    static constexpr int SP_STAGE = SP_A + VG_TILE;
    static constexpr int SP_BAR = 3 * SP_STAGE;
    static constexpr int SP_GATE = SP_BAR + 128;
    static constexpr int SP_SMEM = SP_GATE + (C + 8) * 4 + 1024;
    static_assert(TAYLOR || (SP_A % 1024 == 0 && SP_STAGE % 1024 == 0 && SP_SMEM <= 227 * 1024),
                  "state-pass stages");
};

using BwdCfg128 = BwdCfg<128, 128, false>;
using BwdCfg64 = BwdCfg<64, 64, false>;
using BwdCfgT16 = BwdCfg<16, 64, true>;

struct BwdParams {
    float *dd;            // [BH, N, 2]: den_i, dden_i
    float *ws_s;          // [BH, P, F, NA] state increments per segment
    float *ws_r;          // [BH, P, F, NA] R increments per segment
    void *dq, *dk, *dv;   // [BH, N, D] / [BH, N, DV] bf16
    int N, P, nchunks, cps;
    // Taylor map: 1/d'^(1/4), 1/(sqrt2 sqrt d'), 1/sqrt(d') (pair features and
    // the score's linear term), 1/(2 d') (its square term)
    float inv_c1, inv_c2, inv_c3, k2;
    // gated form (the GATED kernels only): log forget gate g_t per token
    // [BH, N]; each segment's summed gate [BH, P] (written by the S pass);
    // per token [BH, N]: r_i's part over earlier chunks (forward-order pass),
    // then c_j - r_j (reverse pass); and dL/dg [BH, N], its reverse prefix sum, negated
    const float *logdecay;
    float *ws_log, *cvec, *dg;
};

namespace bwd_detail {

using namespace sm100;
using namespace fwd_detail;

// Block barrier that also orders tcgen05 and async-proxy accesses around it.
__device__ __forceinline__ void full_sync()
{
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
}

__device__ __forceinline__ uint32_t pack_f16(float a, float b)
{
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// elu(x)+1 of two bf16 values evaluated in fp32 (its exp through __expf,
// ~2^-21 relative) and rounded to nearest once, as a bf16 pair.  The packed
// bf16 form (elu1_bf16x2: argument and exp2 each in 8-bit bf16) left the
// reverse pass's pair terms ~0.17 % low on average against fp64, while the
// packed fp16 form below showed no such offset; the gated reverse passes sum
// per-token differences of those terms over the whole sequence for dL/dg,
// where a one-sided error accumulates, so they take this form.
__device__ __forceinline__ float elu1_f32(float x) { return x > 0.f ? x + 1.f : __expf(x); }

__device__ __forceinline__ uint32_t elu1_rn_bf16x2(uint32_t x)
{
    return pack_bf16(elu1_f32(__uint_as_float(x << 16)), elu1_f32(__uint_as_float(x & 0xFFFF0000u)));
}

// elu(x)+1 of two bf16 values, as fp16: max(x,0) + 2^(min(x,0) log2 e), the
// exponent argument rounded once to fp16 and the packed exp2 in fp16 (11
// significant bits, so phi - 1 keeps ~8 bits for |x| ~ 0.1).
__device__ __forceinline__ uint32_t elu1_f16x2_from_bf16x2(uint32_t x)
{
    const float lo = __uint_as_float(x << 16), hi = __uint_as_float(x & 0xFFFF0000u);
    const uint32_t arg = pack_f16(fminf(lo, 0.f) * 1.4426950408889634f, fminf(hi, 0.f) * 1.4426950408889634f);
    const uint32_t pos = pack_f16(fmaxf(lo, 0.f), fmaxf(hi, 0.f));
    uint32_t ex, r;
    asm("ex2.approx.f16x2 %0, %1;" : "=r"(ex) : "r"(arg));
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(pos), "r"(ex));
    return r;
}

// elu(x)+1 in place (bf16) on the 64-column block `blk` of row `row` of a
// bf16 SW128 tile; zeros when `zero`.  EXACT: the fp32 form rounded once.
template <bool EXACT>
__device__ __forceinline__ void phi_block_inplace(uint32_t tile, int row, bool zero, int blk)
{
    uint4 raw[8];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) raw[cc] = lds128(tile + sw128_off(row, blk * 64 + cc * 8));
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        uint4 r = raw[cc];
        r = zero ? make_uint4(0u, 0u, 0u, 0u)
                 : EXACT ? make_uint4(elu1_rn_bf16x2(r.x), elu1_rn_bf16x2(r.y), elu1_rn_bf16x2(r.z), elu1_rn_bf16x2(r.w))
                         : make_uint4(elu1_bf16x2(r.x), elu1_bf16x2(r.y), elu1_bf16x2(r.z), elu1_bf16x2(r.w));
        sts128(tile + sw128_off(row, blk * 64 + cc * 8), r);
    }
}

// phi(x) s in place (bf16) on the 64-column block `blk` of row `row` of a bf16
// SW128 tile.  EXACT: phi in fp32 times s, rounded once; otherwise the packed
// bf16 phi times s (two roundings).
template <bool EXACT>
__device__ __forceinline__ void phi_block_scaled(uint32_t tile, int row, float s, int blk)
{
    uint4 raw[8];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) raw[cc] = lds128(tile + sw128_off(row, blk * 64 + cc * 8));
    const uint32_t s2 = pack_bf16(s, s);
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        uint32_t w[4] = {raw[cc].x, raw[cc].y, raw[cc].z, raw[cc].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if constexpr (EXACT) {
                w[e] = pack_bf16(elu1_f32(__uint_as_float(w[e] << 16)) * s,
                                 elu1_f32(__uint_as_float(w[e] & 0xFFFF0000u)) * s);
            } else {
                const uint32_t ph = elu1_bf16x2(w[e]);
                asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(w[e]) : "r"(ph), "r"(s2));
            }
        }
        sts128(tile + sw128_off(row, blk * 64 + cc * 8), make_uint4(w[0], w[1], w[2], w[3]));
    }
}

// Ones column (column DV of V_aug = block DV/16, column 0) for all 128 rows.
__device__ __forceinline__ void write_ones_block(uint8_t *blk, int r)
{
    uint4 *row = reinterpret_cast<uint4 *>(blk + (r >> 3) * 256 + (r & 7) * 32);
    const int c = (r >> 2) & 1;
    row[c] = make_uint4(pack_bf16(1.f, 0.f), 0u, 0u, 0u);
    row[c ^ 1] = make_uint4(0u, 0u, 0u, 0u);
}

// Row r of the augmentation block of G': [dden, 0, ..., 0].
__device__ __forceinline__ void write_dden(uint8_t *blk, int r, float dden)
{
    uint4 *row = reinterpret_cast<uint4 *>(blk + (r >> 3) * 256 + (r & 7) * 32);
    const int c = (r >> 2) & 1;
    row[c] = make_uint4(pack_bf16(dden, 0.f), 0u, 0u, 0u);
    row[c ^ 1] = make_uint4(0u, 0u, 0u, 0u);
}

// 16 fp32 values of row f of an F x NA state as bf16 into a snapshot tile
// (SW32 16-column blocks of F rows); with `lo`, also the rounding remainder
// v - bf16(v) into a second tile, so hi + lo carries ~16 significant bits.
template <int F>
__device__ __forceinline__ void snap_cols(uint32_t a_hi, uint32_t a_lo, int f, int c0, const float *v, bool lo)
{
    float r[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) r[e] = v[e] - __bfloat162float(__float2bfloat16_rn(v[e]));
    sts128(a_hi + sw32_off(f, c0, F), make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                                 pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7])));
    sts128(a_hi + sw32_off(f, c0 + 8, F), make_uint4(pack_bf16(v[8], v[9]), pack_bf16(v[10], v[11]),
                                                     pack_bf16(v[12], v[13]), pack_bf16(v[14], v[15])));
    if (lo) {
        sts128(a_lo + sw32_off(f, c0, F), make_uint4(pack_bf16(r[0], r[1]), pack_bf16(r[2], r[3]),
                                                     pack_bf16(r[4], r[5]), pack_bf16(r[6], r[7])));
        sts128(a_lo + sw32_off(f, c0 + 8, F), make_uint4(pack_bf16(r[8], r[9]), pack_bf16(r[10], r[11]),
                                                         pack_bf16(r[12], r[13]), pack_bf16(r[14], r[15])));
    }
}

// Row f (thread) of a state tile [F x NA] fp32 in TMEM (M = 128 layout) to its
// bf16 snapshot(s).
template <int F, int NA>
__device__ __forceinline__ void snapshot_state(uint32_t tS_lane, uint8_t *snap, uint8_t *snap_lo, int f,
                                               int c_lo = 0, int c_hi = NA)
{
#pragma unroll 1
    for (int c0 = c_lo; c0 < c_hi; c0 += 16) {
        float v[16];
        tmem_ld16(tS_lane + c0, v);
        tmem_ld_wait();
        snap_cols<F>(smem_addr(snap), snap_lo ? smem_addr(snap_lo) : 0u, f, c0, v, snap_lo != nullptr);
    }
}

// Masked scores of one TMEM row (128 fp32 columns at `src`) packed as bf16
// pairs into 64 columns at `dst` (may alias the first half of src).
// keep(j) decides which entries survive the causal mask.
template <typename Keep>
__device__ __forceinline__ void mask_pack_row(uint32_t src, uint32_t dst, Keep keep)
{
#pragma unroll 1
    for (int j0 = 0; j0 < 128; j0 += 64) {
        float a[64];
        tmem_ld32(src + j0, a);
        tmem_ld32(src + j0 + 32, a + 32);
        tmem_ld_wait();
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) pk[e / 2] = pack_bf16(keep(j0 + e) ? a[e] : 0.f, keep(j0 + e + 1) ? a[e + 1] : 0.f);
        tmem_st32(dst + j0 / 2, pk);
    }
    tmem_st_wait();
}


// ---- fp16 operand helpers (the forward-order pass runs its MMAs on fp16)

__device__ __forceinline__ void unpack8_f16(uint4 u, float *f)
{
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 t = __half22float2(h[k]);
        f[2 * k] = t.x;
        f[2 * k + 1] = t.y;
    }
}

__device__ __forceinline__ float f16_rem(float x) { return x - __half2float(__float2half_rn(x)); }

// Two bf16 values -> the same values as fp16 (exact inside the fp16 range).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x)
{
    return pack_f16(__uint_as_float(x << 16), __uint_as_float(x & 0xFFFF0000u));
}

// elu(x)+1 of the 64-column block `blk` of row `row` of a bf16 SW128 tile,
// rewritten in place as fp16 (the forward-order pass's operands); zeros when
// `zero`.
__device__ __forceinline__ void phi_block_f16(uint32_t tile, int row, bool zero, int blk)
{
    uint4 raw[8];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) raw[cc] = lds128(tile + sw128_off(row, blk * 64 + cc * 8));
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        const uint4 r = raw[cc];
        sts128(tile + sw128_off(row, blk * 64 + cc * 8),
               zero ? make_uint4(0u, 0u, 0u, 0u)
                    : make_uint4(elu1_f16x2_from_bf16x2(r.x), elu1_f16x2_from_bf16x2(r.y),
                                 elu1_f16x2_from_bf16x2(r.z), elu1_f16x2_from_bf16x2(r.w)));
    }
}

// mask_pack_row_f16 for two threads per row: the 64 source columns from j0.
// With `aliased` the packed columns may overlap source columns the other
// thread has not read yet, so the block meets at a barrier between the loads
// and the stores (every thread must then call this).
template <typename Keep>
__device__ __forceinline__ void mask_pack_half_f16(uint32_t src, uint32_t dst, int j0, bool aliased, Keep keep)
{
    float a[64];
    tmem_ld32(src + j0, a);
    tmem_ld32(src + j0 + 32, a + 32);
    tmem_ld_wait();
    if (aliased) {
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    uint32_t pk[32];
#pragma unroll
    for (int e = 0; e < 64; e += 2) pk[e / 2] = pack_f16(keep(j0 + e) ? a[e] : 0.f, keep(j0 + e + 1) ? a[e + 1] : 0.f);
    tmem_st32(dst + j0 / 2, pk);
    tmem_st_wait();
}

// Row r of a 16-column SW32 block of 128 rows: [first, 0, ..., 0] in fp16.
__device__ __forceinline__ void write_first_f16(uint8_t *blk, int r, float first)
{
    uint4 *row = reinterpret_cast<uint4 *>(blk + (r >> 3) * 256 + (r & 7) * 32);
    const int c = (r >> 2) & 1;
    row[c] = make_uint4(pack_f16(first, 0.f), 0u, 0u, 0u);
    row[c ^ 1] = make_uint4(0u, 0u, 0u, 0u);
}

// fp16 hi/lo snapshot of 16 state values of row f.
template <int F>
__device__ __forceinline__ void snap_cols_f16(uint32_t a_hi, uint32_t a_lo, int f, int c0, const float *v)
{
    sts128(a_hi + sw32_off(f, c0, F), make_uint4(pack_f16(v[0], v[1]), pack_f16(v[2], v[3]),
                                                 pack_f16(v[4], v[5]), pack_f16(v[6], v[7])));
    sts128(a_hi + sw32_off(f, c0 + 8, F), make_uint4(pack_f16(v[8], v[9]), pack_f16(v[10], v[11]),
                                                     pack_f16(v[12], v[13]), pack_f16(v[14], v[15])));
    sts128(a_lo + sw32_off(f, c0, F), make_uint4(pack_f16(f16_rem(v[0]), f16_rem(v[1])),
                                                 pack_f16(f16_rem(v[2]), f16_rem(v[3])),
                                                 pack_f16(f16_rem(v[4]), f16_rem(v[5])),
                                                 pack_f16(f16_rem(v[6]), f16_rem(v[7]))));
    sts128(a_lo + sw32_off(f, c0 + 8, F), make_uint4(pack_f16(f16_rem(v[8]), f16_rem(v[9])),
                                                     pack_f16(f16_rem(v[10]), f16_rem(v[11])),
                                                     pack_f16(f16_rem(v[12]), f16_rem(v[13])),
                                                     pack_f16(f16_rem(v[14]), f16_rem(v[15]))));
}

template <typename Keep>
__device__ __forceinline__ void mask_pack_row_f16(uint32_t src, uint32_t dst, Keep keep)
{
#pragma unroll 1
    for (int j0 = 0; j0 < 128; j0 += 64) {
        float a[64];
        tmem_ld32(src + j0, a);
        tmem_ld32(src + j0 + 32, a + 32);
        tmem_ld_wait();
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) pk[e / 2] = pack_f16(keep(j0 + e) ? a[e] : 0.f, keep(j0 + e + 1) ? a[e + 1] : 0.f);
        tmem_st32(dst + j0 / 2, pk);
    }
    tmem_st_wait();
}

// mask_pack_row for two threads per row: this thread takes the 64 source
// columns from j0 and writes 32 packed columns at dst + j0/2.  The packed
// columns may alias source columns the other thread has not read yet, so the
// whole block meets at a barrier between the loads and the stores (every
// thread must call this).
template <typename Keep>
__device__ __forceinline__ void mask_pack_half(uint32_t src, uint32_t dst, int j0, Keep keep)
{
    float a[64];
    tmem_ld32(src + j0, a);
    tmem_ld32(src + j0 + 32, a + 32);
    tmem_ld_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    uint32_t pk[32];
#pragma unroll
    for (int e = 0; e < 64; e += 2) pk[e / 2] = pack_bf16(keep(j0 + e) ? a[e] : 0.f, keep(j0 + e + 1) ? a[e + 1] : 0.f);
    tmem_st32(dst + j0 / 2, pk);
    tmem_st_wait();
}

// mask_pack_row_hilo for two threads per row: the 64 source columns from j0
// (destinations do not alias the source).
template <typename Keep>
__device__ __forceinline__ void mask_pack_half_hilo(uint32_t src, uint32_t dst_hi, uint32_t dst_lo, int j0, Keep keep)
{
    float a[64];
    tmem_ld32(src + j0, a);
    tmem_ld32(src + j0 + 32, a + 32);
    tmem_ld_wait();
    uint32_t hi[32], lo[32];
#pragma unroll
    for (int e = 0; e < 64; e += 2) {
        const float x0 = keep(j0 + e) ? a[e] : 0.f, x1 = keep(j0 + e + 1) ? a[e + 1] : 0.f;
        hi[e / 2] = pack_bf16(x0, x1);
        lo[e / 2] = pack_bf16(x0 - __bfloat162float(__float2bfloat16_rn(x0)),
                              x1 - __bfloat162float(__float2bfloat16_rn(x1)));
    }
    tmem_st32(dst_hi + j0 / 2, hi);
    tmem_st32(dst_lo + j0 / 2, lo);
    tmem_st_wait();
}

// Masked scores packed as bf16 hi (at dst_hi) and the bf16 remainder (at
// dst_lo), 64 columns each.
template <typename Keep>
__device__ __forceinline__ void mask_pack_row_hilo(uint32_t src, uint32_t dst_hi, uint32_t dst_lo, Keep keep)
{
#pragma unroll 1
    for (int j0 = 0; j0 < 128; j0 += 64) {
        float a[64];
        tmem_ld32(src + j0, a);
        tmem_ld32(src + j0 + 32, a + 32);
        tmem_ld_wait();
        uint32_t hi[32], lo[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
            const float x0 = keep(j0 + e) ? a[e] : 0.f, x1 = keep(j0 + e + 1) ? a[e + 1] : 0.f;
            hi[e / 2] = pack_bf16(x0, x1);
            lo[e / 2] = pack_bf16(x0 - __bfloat162float(__float2bfloat16_rn(x0)),
                                  x1 - __bfloat162float(__float2bfloat16_rn(x1)));
        }
        tmem_st32(dst_hi + j0 / 2, hi);
        tmem_st32(dst_lo + j0 / 2, lo);
    }
    tmem_st_wait();
}

// ---- state tiles

// Feature row held by lane l of quadrant wq in state tile t, or -1 (M = 128:
// row = lane; M = 64: row 16 wq + l in lane 32 wq + l, l < 16).
template <class Cfg>
__device__ __forceinline__ int state_row(int t, int wq, int l)
{
    const int f = Cfg::tile_m(t) == 128 ? Cfg::tile_f0(t) + 32 * wq + l
                                        : (l < 16 ? Cfg::tile_f0(t) + 16 * wq + l : Cfg::F);
    return f < Cfg::F ? f : -1;
}

// Whether quadrant wq holds a kept row of state tile t (warp-uniform).
template <class Cfg>
__device__ __forceinline__ bool state_quadrant(int t, int wq)
{
    return Cfg::tile_f0(t) + (Cfg::tile_m(t) == 128 ? 32 : 16) * wq < Cfg::F;
}

// bf16 or fp16 pair, as the pass's MMA kind wants.
template <bool F16>
__device__ __forceinline__ uint32_t pack2(float a, float b)
{
    if constexpr (F16) return pack_f16(a, b);
    else return pack_bf16(a, b);
}

// Row r of a 16-column SW32 block of 128 rows: [first, 0, ..., 0].
template <bool F16>
__device__ __forceinline__ void write_first(uint8_t *blk, int r, float first)
{
    if constexpr (F16) write_first_f16(blk, r, first);
    else write_dden(blk, r, first);
}

// Masked scores of this thread's 64 columns from j0, packed as pairs at
// dst + j0/2.  With `aliased` the packed columns may overlap source columns
// the other thread of the row has not read yet, so the whole block meets at
// a barrier between the loads and the stores (every thread must call this).
// With TAY the raw scores s become 1 + s k1 + s^2 k2 first.
template <bool F16, bool TAY, typename Keep>
__device__ __forceinline__ void mask_pack_half_g(uint32_t src, uint32_t dst, int j0, bool aliased, float k1, float k2,
                                                 Keep keep)
{
    float a[64];
    tmem_ld32(src + j0, a);
    tmem_ld32(src + j0 + 32, a + 32);
    tmem_ld_wait();
    if (aliased) {
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if constexpr (TAY) {
#pragma unroll
        for (int e = 0; e < 64; ++e) a[e] = fmaf(a[e], fmaf(a[e], k2, k1), 1.f);
    }
    uint32_t pk[32];
#pragma unroll
    for (int e = 0; e < 64; e += 2) pk[e / 2] = pack2<F16>(keep(j0 + e) ? a[e] : 0.f, keep(j0 + e + 1) ? a[e + 1] : 0.f);
    tmem_st32(dst + j0 / 2, pk);
    tmem_st_wait();
}

// ---- the Taylor map, d' = 16: the folded features packed to 160
//   0: 1;  1..16: x_a / d'^(1/4);  17..32: x_a^2 / (sqrt2 sqrt d');
//   33..152: x_a x_b / sqrt(d'), a < b, row-major pairs;  153..159: 0.

__host__ __device__ constexpr int tay_kind(int f) { return f == 0 ? 0 : f <= 16 ? 1 : f <= 32 ? 2 : f < 153 ? 3 : 4; }
__host__ __device__ constexpr int tay_a(int f)
{
    if (f <= 16) return f - 1;
    if (f <= 32) return f - 17;
    int p = f - 33, a = 0;
    while (p >= 15 - a) {
        p -= 15 - a;
        ++a;
    }
    return a;
}
__host__ __device__ constexpr int tay_b(int f)
{
    int p = f - 33, a = 0;
    while (p >= 15 - a) {
        p -= 15 - a;
        ++a;
    }
    return a + 1 + p;
}

template <int f>
__device__ __forceinline__ float tay_feat(const float *x, const BwdParams &p)
{
    constexpr int kind = tay_kind(f);
    if constexpr (kind == 0) return 1.f;
    else if constexpr (kind == 1) return x[tay_a(f)] * p.inv_c1;
    else if constexpr (kind == 2) return x[tay_a(f)] * x[tay_a(f)] * p.inv_c2;
    else if constexpr (kind == 3) return x[tay_a(f)] * x[tay_b(f)] * p.inv_c3;
    else return 0.f;
}

template <int F0>
__device__ __forceinline__ uint4 tay_feat8(const float *x, const BwdParams &p)
{
    return make_uint4(pack_bf16(tay_feat<F0>(x, p), tay_feat<F0 + 1>(x, p)),
                      pack_bf16(tay_feat<F0 + 2>(x, p), tay_feat<F0 + 3>(x, p)),
                      pack_bf16(tay_feat<F0 + 4>(x, p), tay_feat<F0 + 5>(x, p)),
                      pack_bf16(tay_feat<F0 + 6>(x, p), tay_feat<F0 + 7>(x, p)));
}

template <int FB, int... G>
__device__ __forceinline__ void tay_phi_groups(uint32_t tile, int r, const float *x, bool zero, const BwdParams &p,
                                               std::integer_sequence<int, G...>)
{
    ((sts128(tile + sw128_off(r, FB + 8 * G), zero ? make_uint4(0u, 0u, 0u, 0u) : tay_feat8<FB + 8 * G>(x, p))), ...);
}

// Features [FB, FB + 8 NG) of row r of a phi tile (SW128 blocks of 64
// features), from the raw row x; zeros when `zero`.
template <int FB, int NG>
__device__ __forceinline__ void tay_phi_row(uint32_t tile, int r, const float *x, bool zero, const BwdParams &p)
{
    tay_phi_groups<FB>(tile, r, x, zero, p, std::make_integer_sequence<int, NG>{});
}

// Row r's 16 raw values from a [128 x 16] bf16 SW32 tile.
__device__ __forceinline__ void raw_row16(uint32_t tile, int r, float *x)
{
    unpack8(lds128(tile + sw32_off(r, 0, 128)), x);
    unpack8(lds128(tile + sw32_off(r, 8, 128)), x + 8);
}

// dx += J_phi(x)^T e_f g (the derivative of feature f, weighted by g), and
// sd += g phi_f(x).
template <int f>
__device__ __forceinline__ void tay_vjp_one(float g, const float *x, float *dx, float &sd, const BwdParams &p)
{
    constexpr int kind = tay_kind(f);
    if constexpr (kind == 0) {
        sd += g;
    } else if constexpr (kind == 1) {
        constexpr int a = tay_a(f);
        dx[a] = fmaf(g, p.inv_c1, dx[a]);
        sd = fmaf(g, x[a] * p.inv_c1, sd);
    } else if constexpr (kind == 2) {
        constexpr int a = tay_a(f);
        const float gx = g * x[a] * p.inv_c2;
        dx[a] = fmaf(2.f, gx, dx[a]);
        sd = fmaf(gx, x[a], sd);
    } else if constexpr (kind == 3) {
        constexpr int a = tay_a(f), b = tay_b(f);
        const float gc = g * p.inv_c3;
        dx[a] = fmaf(gc, x[b], dx[a]);
        dx[b] = fmaf(gc, x[a], dx[b]);
        sd = fmaf(gc * x[a], x[b], sd);
    }
}

template <int F0, int... E>
__device__ __forceinline__ void tay_vjp_seq(const float *g, const float *x, float *dx, float &sd, const BwdParams &p,
                                            std::integer_sequence<int, E...>)
{
    (tay_vjp_one<F0 + E>(g[E], x, dx, sd, p), ...);
}

template <int F0>
__device__ __forceinline__ void tay_vjp16(uint32_t tcol, const float *x, float *dx, float &sd, const BwdParams &p)
{
    float g[16];
    tmem_ld16(tcol + F0, g);
    tmem_ld_wait();
    tay_vjp_seq<F0>(g, x, dx, sd, p, std::make_integer_sequence<int, 16>{});
}

template <int FB, int... G>
__device__ __forceinline__ void tay_vjp_groups(uint32_t tcol, const float *x, float *dx, float &sd, const BwdParams &p,
                                               std::integer_sequence<int, G...>)
{
    (tay_vjp16<FB + 16 * G>(tcol, x, dx, sd, p), ...);
}

// J_phi(x)^T dphi over features [80 HALF, 80 HALF + 80), dphi read from TMEM
// columns tcol + f; also sd = dphi . phi(x) over the same features.
template <int HALF>
__device__ __forceinline__ void tay_vjp_half(uint32_t tcol, const float *x, float *dx, float &sd, const BwdParams &p)
{
    tay_vjp_groups<80 * HALF>(tcol, x, dx, sd, p, std::make_integer_sequence<int, 5>{});
}

// The two threads of row i combine their halves of J^T dphi (and of
// dphi . phi) through shared memory; thread hh gets coordinates 8 hh .. 8 hh + 7
// of the whole.  Every thread of the block must call this.
__device__ __forceinline__ void tay_combine(float *xred, float *sred, int hh, int i, const float *dx, float sd,
                                            float *out8, float &sd_all)
{
    float *mine = xred + (hh * 128 + i) * 16;
#pragma unroll
    for (int c = 0; c < 16; c += 4) *reinterpret_cast<float4 *>(mine + c) = make_float4(dx[c], dx[c + 1], dx[c + 2], dx[c + 3]);
    sred[hh * 128 + i] = sd;
    __syncthreads();
    const float *a = xred + i * 16 + 8 * hh, *b = xred + (128 + i) * 16 + 8 * hh;
#pragma unroll
    for (int c = 0; c < 8; ++c) out8[c] = a[c] + b[c];
    sd_all = sred[i] + sred[128 + i];
}


// ---- gated form

// Inclusive prefix sums L_r = g_{t0} + ... + g_{t0+r} of a chunk's log gates
// for row r = 32 wq + l (rows at or past nvalid add 0; a gate below -80
// counts as -80, as in the forward, which keeps every L finite so that no
// difference of two L is inf - inf).  Writes gL[r] (when `writer`) and the
// quadrant totals gL[C + wq]; returns L_r and the chunk's total L_last.
// Every thread of the block calls it (it holds a barrier); the caller
// synchronises again before reading another row's gL.
__device__ __forceinline__ float gate_prefix(const float *g, int r, int nvalid, int wq, int l, bool writer, float *gL,
                                             float &L_last)
{
    float x = r < nvalid ? fmaxf(g[r], -80.f) : 0.f;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, off);
        if (l >= off) x += y;
    }
    if (writer && l == 31) gL[128 + wq] = x;
    __syncthreads();
    float before = 0.f, tot = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < 4; ++w2) {
        const float t = gL[128 + w2];
        if (w2 < wq) before += t;
        tot += t;
    }
    const float L = x + before;
    if (writer) gL[r] = L;
    L_last = tot;
    return L;
}

// TMEM columns [c_lo, c_hi) (multiples of 16) of this thread's lane times s.
__device__ __forceinline__ void tmem_scale(uint32_t t_lane, int c_lo, int c_hi, float s)
{
#pragma unroll 1
    for (int c0 = c_lo; c0 < c_hi; c0 += 16) {
        float v[16];
        tmem_ld16(t_lane + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] *= s;
        tmem_st16(t_lane + c0, v);
    }
    tmem_st_wait();
}

// The state tiles' columns [c_lo, c_hi) of this thread's lane times s.
template <class Cfg>
__device__ __forceinline__ void decay_state_tiles(uint32_t t_state, uint32_t lane, int wq, int c_lo, int c_hi, float s)
{
#pragma unroll
    for (int t = 0; t < Cfg::NT; ++t)
        if (state_quadrant<Cfg>(t, wq)) tmem_scale(t_state + t * Cfg::NA + lane, c_lo, c_hi, s);
}

// Columns [c_lo, c_hi) (multiples of 8) of row r of a 128-row SW32 tile
// (bf16 or fp16 pairs) times s.
template <bool F16>
__device__ __forceinline__ void scale_row_sw32(uint32_t tile, int r, int c_lo, int c_hi, float s)
{
#pragma unroll 1
    for (int c0 = c_lo; c0 < c_hi; c0 += 8) {
        const uint32_t a = tile + sw32_off(r, c0, 128);
        float x[8];
        if constexpr (F16) unpack8_f16(lds128(a), x);
        else unpack8(lds128(a), x);
        sts128(a, make_uint4(pack2<F16>(s * x[0], s * x[1]), pack2<F16>(s * x[2], s * x[3]),
                             pack2<F16>(s * x[4], s * x[5]), pack2<F16>(s * x[6], s * x[7])));
    }
}

// mask_pack_half_g with the gated weights: entry (i, j) of a row, i >= j,
// is also multiplied by exp(L_i - L_j) (the gates a_{j+1} ... a_i); the
// entries masked out are selected away, never multiplied, so an exp that
// overflows there does no harm.  `rowL` is this row's L, `colL` the L of
// column j (shared memory).
template <bool F16, bool TAY, typename Keep>
__device__ __forceinline__ void mask_pack_half_gate(uint32_t src, uint32_t dst, int j0, bool aliased, float k1, float k2,
                                                    float rowL, const float *colL, bool row_is_query, Keep keep)
{
    float a[64];
    tmem_ld32(src + j0, a);
    tmem_ld32(src + j0 + 32, a + 32);
    tmem_ld_wait();
    if (aliased) {
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if constexpr (TAY) {
#pragma unroll
        for (int e = 0; e < 64; ++e) a[e] = fmaf(a[e], fmaf(a[e], k2, k1), 1.f);
    }
#pragma unroll
    for (int e = 0; e < 64; ++e) a[e] *= __expf(row_is_query ? rowL - colL[j0 + e] : colL[j0 + e] - rowL);
    uint32_t pk[32];
#pragma unroll
    for (int e = 0; e < 64; e += 2) pk[e / 2] = pack2<F16>(keep(j0 + e) ? a[e] : 0.f, keep(j0 + e + 1) ? a[e + 1] : 0.f);
    tmem_st32(dst + j0 / 2, pk);
    tmem_st_wait();
}

// mask_pack_half_hilo with the gated weights (reverse pass: row j is a key,
// column i a query, weight exp(L_i - L_j)).
template <typename Keep>
__device__ __forceinline__ void mask_pack_half_hilo_gate(uint32_t src, uint32_t dst_hi, uint32_t dst_lo, int j0,
                                                         float rowL, const float *colL, Keep keep)
{
    float a[64];
    tmem_ld32(src + j0, a);
    tmem_ld32(src + j0 + 32, a + 32);
    tmem_ld_wait();
    uint32_t hi[32], lo[32];
#pragma unroll
    for (int e = 0; e < 64; e += 2) {
        const float x0 = keep(j0 + e) ? a[e] * __expf(colL[j0 + e] - rowL) : 0.f;
        const float x1 = keep(j0 + e + 1) ? a[e + 1] * __expf(colL[j0 + e + 1] - rowL) : 0.f;
        hi[e / 2] = pack_bf16(x0, x1);
        lo[e / 2] = pack_bf16(x0 - __bfloat162float(__float2bfloat16_rn(x0)),
                              x1 - __bfloat162float(__float2bfloat16_rn(x1)));
    }
    tmem_st32(dst_hi + j0 / 2, hi);
    tmem_st32(dst_lo + j0 / 2, lo);
    tmem_st_wait();
}


__device__ __forceinline__ float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// Columns [c_lo, c_hi) (multiples of 8) of row r of a bf16 head tile and its
// bf16 remainder tile (128-row SW32): (head + remainder) times s, split again
// into a head and a remainder.
__device__ __forceinline__ void scale_row_hilo(uint32_t thi, uint32_t tlo, int r, int c_lo, int c_hi, float s)
{
#pragma unroll 1
    for (int c0 = c_lo; c0 < c_hi; c0 += 8) {
        const uint32_t off = sw32_off(r, c0, 128);
        float h[8], lo[8];
        unpack8(lds128(thi + off), h);
        unpack8(lds128(tlo + off), lo);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            h[e] = (h[e] + lo[e]) * s;
            lo[e] = h[e] - bf16_round(h[e]);
        }
        sts128(thi + off, make_uint4(pack_bf16(h[0], h[1]), pack_bf16(h[2], h[3]), pack_bf16(h[4], h[5]), pack_bf16(h[6], h[7])));
        sts128(tlo + off,
               make_uint4(pack_bf16(lo[0], lo[1]), pack_bf16(lo[2], lo[3]), pack_bf16(lo[4], lo[5]), pack_bf16(lo[6], lo[7])));
    }
}

// Column sums over a warp's 32 rows of a 32-column block held one row per
// lane (v[c] = row lane's column c; v is overwritten): lane l returns the sum
// of column l.  A reduce-scatter in five exchange steps (31 shuffles).
__device__ __forceinline__ float warp_colsum32(float *v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const bool up = (lane & w) != 0;
#pragma unroll
        for (int e = 0; e < w; ++e) {
            const float send = up ? v[e] : v[e + w];
            const float keep = up ? v[e + w] : v[e];
            v[e] = keep + __shfl_xor_sync(0xffffffffu, send, w);
        }
    }
    return v[0];
}

// Reverse pass, gated: P^T and dP^T of this thread's 64 columns from j0 in one
// step (row j is a key, column i a query; weight exp(L_i - L_j); with TAY the
// raw scores s become 1 + s k1 + s^2 k2 first).  Also the pair terms
// M_ij = dL/dw_ij w_ij of the chunk from the fp32 scores and dA^T: returns the
// row's part of c_j = sum_i M_ij, and writes the warp's part of each
// column's r_i = sum_j M_ij to rsum[i] (the two come from the same products,
// so the chunk's pairs cancel exactly in the suffix sums of r - c).  P^T
// overwrites the scores' columns, so the block meets at a barrier between
// loading and storing (every thread must call this).
template <bool TAY, typename Keep>
__device__ __forceinline__ float mask_pack_both_gate(uint32_t tA, uint32_t tX, uint32_t tPL, int j0, float k1, float k2,
                                                     float rowL, const float *colL, float *rsum, Keep keep)
{
    float w[64];
    tmem_ld32(tA + j0, w);
    tmem_ld32(tA + j0 + 32, w + 32);
    tmem_ld_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
#pragma unroll
    for (int e = 0; e < 64; ++e) {
        float a = w[e];
        if constexpr (TAY) a = fmaf(a, fmaf(a, k2, k1), 1.f);
        w[e] = keep(j0 + e) ? a * __expf(colL[j0 + e] - rowL) : 0.f;
    }
    {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) pk[e / 2] = pack_bf16(w[e], w[e + 1]);
        tmem_st32(tA + j0 / 2, pk);
    }
    float c = 0.f;
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        float d[32];
        tmem_ld32(tX + j0 + 32 * h2, d);
        tmem_ld_wait();
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            const int i0 = j0 + 32 * h2 + e;
            const float x0 = keep(i0) ? d[e] * __expf(colL[i0] - rowL) : 0.f;
            const float x1 = keep(i0 + 1) ? d[e + 1] * __expf(colL[i0 + 1] - rowL) : 0.f;
            hi[e / 2] = pack_bf16(x0, x1);
            lo[e / 2] = pack_bf16(x0 - __bfloat162float(__float2bfloat16_rn(x0)),
                                  x1 - __bfloat162float(__float2bfloat16_rn(x1)));
        }
        tmem_st16(tA + 64 + (j0 + 32 * h2) / 2, reinterpret_cast<const float *>(hi));
        tmem_st16(tPL + (j0 + 32 * h2) / 2, reinterpret_cast<const float *>(lo));
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            d[e] *= w[32 * h2 + e];   // M_ij (0 where masked)
            c += d[e];
        }
        rsum[j0 + 32 * h2 + (threadIdx.x & 31)] = warp_colsum32(d);
    }
    tmem_st_wait();
    return c;
}

// phi(x) . (X + dr) over features [80 HALF, 80 HALF + 80) of the Taylor map,
// X read from TMEM columns tcol + f, phi from the raw row x; dr_f (the bf16
// remainder of R's normaliser column) only with DR.
template <bool DR, int F0, int... E>
__device__ __forceinline__ float tay_dot_seq(const float *g, const float *x, const float *dr, const BwdParams &p,
                                             std::integer_sequence<int, E...>)
{
    float acc = 0.f;
    ((acc = fmaf(DR ? g[E] + dr[F0 + E] : g[E], tay_feat<F0 + E>(x, p), acc)), ...);
    return acc;
}
template <bool DR, int F0>
__device__ __forceinline__ float tay_dot16(uint32_t tcol, const float *x, const float *dr, const BwdParams &p)
{
    float g[16];
    tmem_ld16(tcol + F0, g);
    tmem_ld_wait();
    return tay_dot_seq<DR, F0>(g, x, dr, p, std::make_integer_sequence<int, 16>{});
}
template <bool DR, int FB, int... G>
__device__ __forceinline__ float tay_dot_groups(uint32_t tcol, const float *x, const float *dr, const BwdParams &p,
                                                std::integer_sequence<int, G...>)
{
    return (tay_dot16<DR, FB + 16 * G>(tcol, x, dr, p) + ...);
}
template <bool DR, int HALF>
__device__ __forceinline__ float tay_dot_half(uint32_t tcol, const float *x, const float *dr, const BwdParams &p)
{
    return tay_dot_groups<DR, 80 * HALF>(tcol, x, dr, p, std::make_integer_sequence<int, 5>{});
}

// phi_j . (X_j + dr) over feature columns [c_lo, c_hi) of an elu phi tile
// (row j; fp16 or bf16 as F16), X from TMEM columns tcol + f; dr only with DR.
template <bool F16, bool DR>
__device__ __forceinline__ float elu_dot_cols(uint32_t tcol, uint32_t phi_tile, int j, int c_lo, int c_hi,
                                              const float *dr)
{
    float acc = 0.f;
#pragma unroll 1
    for (int c0 = c_lo; c0 < c_hi; c0 += 16) {
        float g[16], ph[16];
        tmem_ld16(tcol + c0, g);
        tmem_ld_wait();
        if constexpr (F16) {
            unpack8_f16(lds128(phi_tile + sw128_off(j, c0)), ph);
            unpack8_f16(lds128(phi_tile + sw128_off(j, c0 + 8)), ph + 8);
        } else {
            unpack8(lds128(phi_tile + sw128_off(j, c0)), ph);
            unpack8(lds128(phi_tile + sw128_off(j, c0 + 8)), ph + 8);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) acc = fmaf(DR ? g[e] + dr[c0 + e] : g[e], ph[e], acc);
    }
    return acc;
}

}  // namespace bwd_detail

// ---------------------------------------------------------------------------
// Forward-order pass: dq, and den_i, dden_i per token.
//
// elu: the MMAs run on fp16 operands (A and B both fp16), not bf16: dq is
// carried by phi - 1, which is ~0.1 for small inputs, and bf16 keeps only ~5
// bits of it (relative error ~2/|phi - 1| x 2^-9 in dq); fp16 keeps 3 more.
// V is converted exactly; the state snapshot and G'' keep an extra remainder
// for the inter-chunk term, and dphi(q) is projected orthogonal to phi(q).
// Taylor: the same steps on bf16 operands, with the raw scores and the
// feature-to-coordinate chain rule described at the top of the file.
template <class Cfg, bool GATED = false>
__global__ void __launch_bounds__(256, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_dq, const BwdParams p)
{
    using namespace bwd_detail;
    constexpr int C = Cfg::C, D = Cfg::D, DV = Cfg::DV, NA = Cfg::NA, F = Cfg::F, NT = Cfg::NT;
    constexpr bool TAY = Cfg::TAYLOR, F16 = Cfg::F16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *mma_bar = tma_bar + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_bar + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tma_bar + 3);
    // 256 threads: warps w and w + 4 share the TMEM lanes of rows 32 (w % 4) ..
    // + 31 and split every per-row step by columns; row sums meet in red[]
    const int tid = threadIdx.x, warp = tid >> 5, wq = warp & 3, hh = warp >> 2, l = tid & 31;
    const int row = wq * 32 + l;
    float *red = reinterpret_cast<float *>(smem + Cfg::OFF_RED);   // [3][2][C], then (Taylor) [2][C][16]
    const int bh = blockIdx.x / p.P, seg = blockIdx.x % p.P;
    const int c_begin = seg * p.cps, c_end = min(p.nchunks, c_begin + p.cps);
    const int N = p.N;
    uint8_t *sQ = smem + Cfg::OFF_Q, *sK = smem + Cfg::OFF_K, *sV = smem + Cfg::OFF_V, *sG = smem + Cfg::OFF_G,
            *sS = smem + Cfg::OFF_S, *sSL = smem + Cfg::OFF_SL;
    const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV), aG = smem_addr(sG), aS = smem_addr(sS),
                   aSL = smem_addr(sSL), aRQ = smem_addr(smem + Cfg::OFF_RQ), aRK = smem_addr(smem + Cfg::OFF_RK);

    if (tid == 0) {
        mbar_init(tma_bar, 1);
        mbar_init(mma_bar, 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 0) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    if (hh == 0) write_first<F16>(sV + (DV / 16) * Cfg::BLK, row, 1.f);   // ones column of V_aug
    if constexpr (TAY) {
        // features 160..191 of both phi tiles stay zero (the M = 64 state tile reads them)
#pragma unroll
        for (int f0 = F; f0 < Cfg::FT; f0 += 8)
            sts128((hh ? aK : aQ) + sw128_off(row, f0), make_uint4(0u, 0u, 0u, 0u));
    }
    __syncthreads();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane = (uint32_t)(wq * 32) << 16;
    const int na_lo = hh ? Cfg::NA_SPLIT : 0, na_hi = hh ? NA : Cfg::NA_SPLIT;   // this thread's columns of S_aug
    const uint32_t tA = tmem, tX = tmem + Cfg::COL_X, tS = tmem + Cfg::COL_S, tGL = tmem + Cfg::COL_GL;
    auto snap = [&](int f, int c0, const float *v) {
        if constexpr (F16) snap_cols_f16<F>(aS, aSL, f, c0, v);
        else snap_cols<F>(aS, aSL, f, c0, v, true);
    };
    float *gL = reinterpret_cast<float *>(smem + Cfg::OFF_GATE);   // gated: the chunk's prefix sums of the gates

    // ---- state entering the segment: sum of the earlier segments' increments
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        if (!state_quadrant<Cfg>(t, wq)) continue;
        const int f = state_row<Cfg>(t, wq, l);
        for (int c0 = na_lo; c0 < na_hi; c0 += 16) {
            float v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0.f;
            if (f >= 0)
                for (int s2 = 0; s2 < seg; ++s2) {
                    const float *src = p.ws_s + ((size_t)(bh * p.P + s2) * F + f) * NA + c0;
                    if constexpr (GATED) {
                        // the state after segment s2 is its increment plus the earlier
                        // state decayed by the segment's gates
                        const float d = __expf(p.ws_log[(size_t)bh * p.P + s2]);
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = fmaf(v[e], d, src[e]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] += src[e];
                    }
                }
            tmem_st16(tS + t * NA + lane + c0, v);
            if (f >= 0) snap(f, c0, v);
        }
    }
    tmem_st_wait();
    full_sync();

    uint32_t tph = 0, mph = 0;
    for (int chunk = c_begin; chunk < c_end && !*abort_flag; ++chunk) {
        const int t0 = chunk * C, i = row;
        const bool valid = t0 + i < N;
        if (tid == 0) {
            // the previous chunk's dq left from the Q tile (its raw tile for Taylor)
            if (chunk > c_begin) bulk_wait_read();
            mbar_arrive_expect_tx(tma_bar, TAY ? 2 * Cfg::RAW + 2 * C * DV * 2 : 2 * C * D * 2 + 2 * C * DV * 2);
            if constexpr (TAY) {
                tma_load_3d(smem + Cfg::OFF_RQ, &tm_q, tma_bar, 0, t0, bh);
                tma_load_3d(smem + Cfg::OFF_RK, &tm_k, tma_bar, 0, t0, bh);
            } else {
                for (int x = 0; x < D; x += 64) {
                    tma_load_3d(sQ + (x / 64) * C * 128, &tm_q, tma_bar, x, t0, bh);
                    tma_load_3d(sK + (x / 64) * C * 128, &tm_k, tma_bar, x, t0, bh);
                }
            }
            for (int x = 0; x < DV; x += 16) {
                tma_load_3d(sV + (x / 16) * Cfg::BLK, &tm_v, tma_bar, x, t0, bh);
                tma_load_3d(sG + (x / 16) * Cfg::BLK, &tm_do, tma_bar, x, t0, bh);
            }
        }
        if (!mbar_wait(tma_bar, tph)) *abort_flag = 1;
        tph ^= 1u;
        // gated: L_i = g_{t0} + ... + g_i over the chunk; exp(L_i) scales the
        // carried state's terms of row i, exp(L_last - L_j) the state update by key j
        float Lrow = 0.f, Llast = 0.f;
        if constexpr (GATED) {
            Lrow = gate_prefix(p.logdecay + (size_t)bh * N + t0, row, min(C, N - t0), wq, l, hh == 0, gL, Llast);
            if (hh == 0) write_first<F16>(sV + (DV / 16) * Cfg::BLK, row, 1.f);   // scaled by the last chunk's update
        }
        if constexpr (TAY) {
            // phi(Q), phi(K): this thread's 80 of the 160 features of row i
            float xq[16], xk[16];
            raw_row16(aRQ, i, xq);
            raw_row16(aRK, i, xk);
            if (hh == 0) {
                tay_phi_row<0, 10>(aQ, i, xq, false, p);
                tay_phi_row<0, 10>(aK, i, xk, !valid, p);
            } else {
                tay_phi_row<80, 10>(aQ, i, xq, false, p);
                tay_phi_row<80, 10>(aK, i, xk, !valid, p);
            }
        } else {
            // fp16 operands: phi(Q), phi(K) in place; V converted in place
            if (D == 128) {
                phi_block_f16(aQ, i, false, hh);
                phi_block_f16(aK, i, !valid, hh);
            } else if (hh == 0) {
                phi_block_f16(aQ, i, false, 0);
            } else {
                phi_block_f16(aK, i, !valid, 0);
            }
#pragma unroll
            for (int c0 = hh * (DV / 2); c0 < (hh + 1) * (DV / 2); c0 += 8) {
                const uint32_t a = aV + sw32_off(i, c0, C);
                const uint4 r = lds128(a);
                sts128(a, make_uint4(bf16x2_to_f16x2(r.x), bf16x2_to_f16x2(r.y), bf16x2_to_f16x2(r.z),
                                     bf16x2_to_f16x2(r.w)));
            }
        }
        full_sync();
        if (*abort_flag) break;

        // scores
        if (tid == 0) {
            if constexpr (TAY) {
                mma_bf16(tA, smem_desc(aRQ, 16, 256, kSw32), smem_desc(aRK, 16, 256, kSw32), idesc_bf16(128, 128, 0, 0),
                         false);
            } else {
#pragma unroll
                for (int kk = 0; kk < F / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (C * 128) + (kk & 3) * 32;
                    mma_bf16(tA, smem_desc(aQ + off, 16, 1024, kSw128), smem_desc(aK + off, 16, 1024, kSw128),
                             idesc_f16(128, 128, 0, 0), kk > 0);
                }
            }
            mma_commit(mma_bar);
        }
        if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
        mph ^= 1u;
        tc_fence_after();
        if constexpr (GATED)
            mask_pack_half_gate<F16, TAY>(tA + lane, tA + lane, 64 * hh, true, p.inv_c3, p.k2, Lrow, gL, true,
                                          [&](int j) { return j <= i; });
        else
            mask_pack_half_g<F16, TAY>(tA + lane, tA + lane, 64 * hh, true, p.inv_c3, p.k2, [&](int j) { return j <= i; });
        full_sync();

        // O_aug = P V_aug + phi(Q) S_aug  (gated: the state term first, scaled
        // per row by exp(L_i), then the chunk's own term added)
        if constexpr (GATED) {
            if (tid == 0) {
                const uint32_t id_o = F16 ? idesc_f16(128, NA, 0, 1) : idesc_bf16(128, NA, 0, 1);
#pragma unroll
                for (int kk = 0; kk < F / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (C * 128) + (kk & 3) * 32;
                    mma_bf16(tX, smem_desc(aQ + off, 16, 1024, kSw128), smem_desc(aS + kk * 512, Cfg::S_BLK, 256, kSw32),
                             id_o, kk > 0);
                    // and its remainder: y_i, hence dden_i, to ~16 bits (dden_i enters
                    // every pair term of row i in dL/dg)
                    mma_bf16(tX, smem_desc(aQ + off, 16, 1024, kSw128), smem_desc(aSL + kk * 512, Cfg::S_BLK, 256, kSw32),
                             id_o, true);
                }
                mma_commit(mma_bar);
            }
            if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
            mph ^= 1u;
            tc_fence_after();
            tmem_scale(tX + lane, na_lo, na_hi, __expf(Lrow));
            full_sync();
        }
        if (tid == 0) {
            const uint32_t id_o = F16 ? idesc_f16(128, NA, 0, 1) : idesc_bf16(128, NA, 0, 1);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                mma_bf16_ts(tX, tA + kk * 8, smem_desc(aV + kk * 512, Cfg::BLK, 256, kSw32), id_o, GATED || kk > 0);
            if constexpr (!GATED) {
#pragma unroll
                for (int kk = 0; kk < F / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (C * 128) + (kk & 3) * 32;
                    mma_bf16(tX, smem_desc(aQ + off, 16, 1024, kSw128),
                             smem_desc(aS + kk * 512, Cfg::S_BLK, 256, kSw32), id_o, true);
                }
            }
            mma_commit(mma_bar);
        }
        if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
        mph ^= 1u;
        tc_fence_after();

        // y, den; G'' = den * G' = [dO | -dO . y] in place over dO (with its
        // remainder in TMEM).  Working with den * g keeps every operand in
        // fp16's normal range (g itself is ~|dO| / (F i)); the rows of dphi(Q) are
        // divided by den at the end.  den_i and dden_i = -(dO . y)/den go to the
        // workspace for the reverse pass.
        float den_row;
        {
            float dv16[16];
            tmem_ld16(tX + lane + DV, dv16);
            tmem_ld_wait();
            const float den = dv16[0];
            den_row = den;
            const float inv = valid ? 1.f / den : 0.f;
            float gy = 0.f;   // dO . y over this thread's half of the columns
            {
                const int half = (DV / 2) * hh;
                uint32_t glo[DV / 4];
#pragma unroll
                for (int u = 0; u < DV / 32; ++u) {
                    const int c0 = half + 16 * u;
                    float num[16], go[16];
                    tmem_ld16(tX + lane + c0, num);
                    tmem_ld_wait();
                    const uint32_t a0 = aG + sw32_off(i, c0, C), a1 = aG + sw32_off(i, c0 + 8, C);
                    unpack8(lds128(a0), go);
                    unpack8(lds128(a1), go + 8);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        if (!valid) go[e] = 0.f;
                        gy = fmaf(go[e], num[e] * inv, gy);
                    }
                    sts128(a0, make_uint4(pack2<F16>(go[0], go[1]), pack2<F16>(go[2], go[3]), pack2<F16>(go[4], go[5]),
                                          pack2<F16>(go[6], go[7])));
                    sts128(a1, make_uint4(pack2<F16>(go[8], go[9]), pack2<F16>(go[10], go[11]),
                                          pack2<F16>(go[12], go[13]), pack2<F16>(go[14], go[15])));
#pragma unroll
                    for (int e = 0; e < 16; e += 2) {
                        if constexpr (F16) {
                            glo[(16 * u + e) / 2] = pack_f16(f16_rem(go[e]), f16_rem(go[e + 1]));
                        } else {
                            glo[(16 * u + e) / 2] = pack_bf16(go[e] - __bfloat162float(__float2bfloat16_rn(go[e])),
                                                              go[e + 1] - __bfloat162float(__float2bfloat16_rn(go[e + 1])));
                        }
                    }
                }
                if constexpr (DV / 4 == 32) tmem_st32(tGL + lane + half / 2, glo);
                else tmem_st16(tGL + lane + half / 2, reinterpret_cast<const float *>(glo));
            }
            red[hh * C + i] = gy;
            __syncthreads();
            gy = red[i] + red[C + i];
            const float ddu = valid ? -gy : 0.f;   // den * dden
            if (hh == 0) {
                write_first<F16>(sG + (DV / 16) * Cfg::BLK, i, ddu);
                uint32_t tail[8];
                if constexpr (F16) tail[0] = pack_f16(f16_rem(ddu), 0.f);
                else tail[0] = pack_bf16(ddu - __bfloat162float(__float2bfloat16_rn(ddu)), 0.f);
#pragma unroll
                for (int e = 1; e < 8; ++e) tail[e] = 0u;
                tmem_st8(tGL + lane + DV / 2, tail);
                if (valid) {
                    p.dd[((size_t)bh * N + t0 + i) * 2] = den;
                    p.dd[((size_t)bh * N + t0 + i) * 2 + 1] = ddu * inv;
                }
            }
            tmem_st_wait();
        }
        full_sync();

        // dA = G'' V_aug^T  (K = the NA augmented columns).  bf16: the
        // remainder of G'' too, so that dA_ij = dO_i . (v_j - y_i) keeps ~16 bits
        // where its two terms cancel (with one token, y_1 = v_1 and dA_11 = 0)
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < NA / 16; ++kk)
                mma_bf16(tX, smem_desc(aG + kk * Cfg::BLK, 16, 256, kSw32), smem_desc(aV + kk * Cfg::BLK, 16, 256, kSw32),
                         F16 ? idesc_f16(128, 128, 0, 0) : idesc_bf16(128, 128, 0, 0), kk > 0);
            if constexpr (!F16) {
#pragma unroll
                for (int kk = 0; kk < NA / 16; ++kk)
                    mma_bf16_ts(tX, tGL + kk * 8, smem_desc(aV + kk * Cfg::BLK, 16, 256, kSw32),
                                idesc_bf16(128, 128, 0, 0), true);
            }
            mma_commit(mma_bar);
        }
        if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
        mph ^= 1u;
        tc_fence_after();
        if constexpr (GATED) {
            mask_pack_half_gate<F16, false>(tX + lane, tA + lane + 64, 64 * hh, false, 0.f, 0.f, Lrow, gL, true,
                                            [&](int j) { return j <= i; });
            // V_aug's last use below is the state update: scale key row i by
            // exp(L_last - L_i) (its ones column too), and decay the state by the
            // chunk's whole gate
            const float w = __expf(Llast - Lrow);
            scale_row_sw32<F16>(aV, i, hh * (DV / 2), (hh + 1) * (DV / 2), w);
            if (hh == 0) write_first<F16>(sV + (DV / 16) * Cfg::BLK, i, w);
            decay_state_tiles<Cfg>(tS, lane, wq, na_lo, na_hi, __expf(Llast));
        } else {
            mask_pack_half_g<F16, false>(tX + lane, tA + lane + 64, 64 * hh, false, 0.f, 0.f,
                                         [&](int j) { return j <= i; });
        }
        full_sync();
        if constexpr (GATED) {
            // the carried state's term of dphi(Q) first, scaled per row by exp(L_i)
            if (tid == 0) {
                const uint32_t id_fk = F16 ? idesc_f16(128, F, 0, 0) : idesc_bf16(128, F, 0, 0);
#pragma unroll
                for (int kk = 0; kk < NA / 16; ++kk) {
                    mma_bf16(tX, smem_desc(aG + kk * Cfg::BLK, 16, 256, kSw32),
                             smem_desc(aS + kk * Cfg::S_BLK, 16, 256, kSw32), id_fk, kk > 0);
                    mma_bf16(tX, smem_desc(aG + kk * Cfg::BLK, 16, 256, kSw32),
                             smem_desc(aSL + kk * Cfg::S_BLK, 16, 256, kSw32), id_fk, true);
                    mma_bf16_ts(tX, tGL + kk * 8, smem_desc(aS + kk * Cfg::S_BLK, 16, 256, kSw32), id_fk, true);
                }
                mma_commit(mma_bar);
            }
            if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
            mph ^= 1u;
            tc_fence_after();
            // r_i's part over the earlier chunks' keys: sum over j < t0 of
            // dL/dw_ij w_ij = phi(q_i) . (their term of dphi(q_i)), to cvec
            float dot;
            if constexpr (TAY) {
                float xq[16];
                raw_row16(aRQ, i, xq);
                dot = hh == 0 ? tay_dot_half<false, 0>(tX + lane, xq, nullptr, p)
                              : tay_dot_half<false, 1>(tX + lane, xq, nullptr, p);
            } else {
                dot = elu_dot_cols<F16, false>(tX + lane, aQ, i, hh * (F / 2), (hh + 1) * (F / 2), nullptr);
            }
            red[hh * C + i] = dot;
            tmem_scale(tX + lane, hh * (F / 2), (hh + 1) * (F / 2), __expf(Lrow));
            full_sync();
            if (hh == 0 && valid) p.cvec[(size_t)bh * N + t0 + i] = (red[i] + red[C + i]) * __expf(Lrow) / den_row;
        }

        // dphi(Q) = dP phi(K) + G'' S_aug^T ;  then S_aug += phi(K)^T V_aug
        if (tid == 0) {
            const uint32_t id_f = F16 ? idesc_f16(128, F, 0, 1) : idesc_bf16(128, F, 0, 1);
            const uint32_t id_fk = F16 ? idesc_f16(128, F, 0, 0) : idesc_bf16(128, F, 0, 0);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                mma_bf16_ts(tX, tA + 64 + kk * 8, smem_desc(aK + kk * 2048, C * 128, 1024, kSw128), id_f,
                            GATED || kk > 0);
            // inter-chunk term in ~16-bit precision: G''_hi S_hi^T + G''_hi S_lo^T + G''_lo S_hi^T
            // (gated: issued above)
#pragma unroll
            for (int kk = 0; kk < (GATED ? 0 : NA / 16); ++kk) {
                mma_bf16(tX, smem_desc(aG + kk * Cfg::BLK, 16, 256, kSw32), smem_desc(aS + kk * Cfg::S_BLK, 16, 256, kSw32),
                         id_fk, true);
                mma_bf16(tX, smem_desc(aG + kk * Cfg::BLK, 16, 256, kSw32), smem_desc(aSL + kk * Cfg::S_BLK, 16, 256, kSw32),
                         id_fk, true);
                mma_bf16_ts(tX, tGL + kk * 8, smem_desc(aS + kk * Cfg::S_BLK, 16, 256, kSw32), id_fk, true);
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int m = Cfg::tile_m(t);
                const uint32_t a_base = aK + (Cfg::tile_f0(t) / 64) * (C * 128);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tS + t * NA, smem_desc(a_base + kk * 2048, C * 128, 1024, kSw128),
                             smem_desc(aV + kk * 512, Cfg::BLK, 256, kSw32),
                             F16 ? idesc_f16(m, NA, 1, 1) : idesc_bf16(m, NA, 1, 1), true);
            }
            mma_commit(mma_bar);
        }
        if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
        mph ^= 1u;
        tc_fence_after();

        // dq = J_phi(q)^T dphi(Q), with dphi(q_i) first projected onto the
        // complement of phi(q_i): y_i is homogeneous of degree 0 in phi(q_i), so
        // the exact dphi(q_i) is orthogonal to phi(q_i); the rounded operands of
        // the MMAs above leave an error mostly along phi(q_i) (elu features are
        // near 1 and the terms cancel), which the projection removes.
        {
            const float rden = valid ? 1.f / den_row : 0.f;
            if constexpr (TAY) {
                float x[16], dx[16], sd = 0.f;
                raw_row16(aRQ, i, x);
#pragma unroll
                for (int c = 0; c < 16; ++c) dx[c] = 0.f;
                if (hh == 0) tay_vjp_half<0>(tX + lane, x, dx, sd, p);
                else tay_vjp_half<1>(tX + lane, x, dx, sd, p);
                float d8[8], sd_all;
                tay_combine(red + 6 * C, red + 2 * C, hh, i, dx, sd, d8, sd_all);
                float xx = 0.f;
#pragma unroll
                for (int c = 0; c < 16; ++c) xx = fmaf(x[c], x[c], xx);
                // |phi|^2 = 1 + |x|^2/sqrt(d') + |x|^4/(2d');  J^T phi = x (1/sqrt(d') + |x|^2/d')
                const float sn = fmaf(xx, fmaf(xx, p.k2, p.inv_c3), 1.f);
                const float proj = sd_all / sn, jt = fmaf(xx, 2.f * p.k2, p.inv_c3);
#pragma unroll
                for (int c = 0; c < 8; ++c) d8[c] = (d8[c] - proj * jt * x[8 * hh + c]) * rden;
                // dq over its own raw q in the raw Q tile (both threads of the row
                // read it before tay_combine's barrier); one TMA store per chunk
                sts128(aRQ + sw32_off(i, 8 * hh, 128), make_uint4(pack_bf16(d8[0], d8[1]), pack_bf16(d8[2], d8[3]),
                                                                  pack_bf16(d8[4], d8[5]), pack_bf16(d8[6], d8[7])));
            } else {
                float sd = 0.f, sn = 0.f;
#pragma unroll 1
                for (int c0 = hh * (F / 2); c0 < (hh + 1) * (F / 2); c0 += 16) {
                    float g[16], ph[16];
                    tmem_ld16(tX + lane + c0, g);
                    tmem_ld_wait();
                    unpack8_f16(lds128(aQ + sw128_off(i, c0)), ph);
                    unpack8_f16(lds128(aQ + sw128_off(i, c0 + 8)), ph + 8);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        sd = fmaf(g[e], ph[e], sd);
                        sn = fmaf(ph[e], ph[e], sn);
                    }
                }
                red[2 * C + hh * C + i] = sd;
                red[4 * C + hh * C + i] = sn;
                __syncthreads();
                sd = red[2 * C + i] + red[3 * C + i];
                sn = red[4 * C + i] + red[5 * C + i];
                const float proj = sd / sn;
#pragma unroll 1
                for (int c0 = hh * (F / 2); c0 < (hh + 1) * (F / 2); c0 += 16) {
                    float g[16], ph[16];
                    tmem_ld16(tX + lane + c0, g);
                    tmem_ld_wait();
                    unpack8_f16(lds128(aQ + sw128_off(i, c0)), ph);
                    unpack8_f16(lds128(aQ + sw128_off(i, c0 + 8)), ph + 8);
#pragma unroll
                    for (int e = 0; e < 16; ++e) g[e] = (g[e] - proj * ph[e]) * fminf(ph[e], 1.f) * rden;
                    // dq over the thread's own phi(q) entries (same SW128 layout); one
                    // TMA store per chunk
#pragma unroll
                    for (int e = 0; e < 16; e += 8)
                        sts128(aQ + sw128_off(i, c0 + e),
                               make_uint4(pack_bf16(g[e], g[e + 1]), pack_bf16(g[e + 2], g[e + 3]),
                                          pack_bf16(g[e + 4], g[e + 5]), pack_bf16(g[e + 6], g[e + 7])));
                }
            }
            if (chunk + 1 < c_end) {
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    if (!state_quadrant<Cfg>(t, wq)) continue;
                    const int f = state_row<Cfg>(t, wq, l);
#pragma unroll 1
                    for (int c0 = na_lo; c0 < na_hi; c0 += 16) {
                        float v[16];
                        tmem_ld16(tS + t * NA + lane + c0, v);
                        tmem_ld_wait();
                        if (f >= 0) snap(f, c0, v);
                    }
                }
            }
        }
        full_sync();
        // the chunk's dq (over phi(Q), or over the raw Q tile for Taylor) leaves
        // by TMA; rows past the slice's end are clipped by the tensor map
        if (tid == 0 && !*abort_flag) {
            if constexpr (TAY) tma_store_3d(&tm_dq, smem + Cfg::OFF_RQ, 0, t0, bh);
            else
                for (int x = 0; x < D; x += 64) tma_store_3d(&tm_dq, sQ + (x / 64) * C * 128, x, t0, bh);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait_all();
    full_sync();
    if (warp == 0) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

// ---------------------------------------------------------------------------
// State increments for the forward-order pass, Taylor map: for each segment
// but the last, sum over its tokens of phi(k_j) [v_j | 1]^T (bf16 operands,
// like the pass that consumes them).  128 threads, one per row, two load
// stages; the phi(K) tile is built from the raw tile of the stage.
template <class Cfg, bool GATED = false>
__global__ void __launch_bounds__(128, 1)
bwd_sstate_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const BwdParams p)
{
    using namespace bwd_detail;
    static_assert(Cfg::TAYLOR, "the elu shapes take bwd_sstate3_kernel");
    constexpr int C = Cfg::C, DV = Cfg::DV, NA = Cfg::NA, F = Cfg::F, NT = Cfg::NT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *mma_bar = tma_bar + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_bar + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tma_bar + 3);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int bh = blockIdx.x / p.P, seg = blockIdx.x % p.P;
    if (seg == p.P - 1) return;   // the last segment's increment is never read
    const int c_begin = seg * p.cps, c_end = min(p.nchunks, c_begin + p.cps);
    const int N = p.N;
    // two stages of [raw K | V_aug], and one phi(K) tile in the K region
    uint8_t *sKs[2] = {smem + Cfg::OFF_RK, smem + Cfg::OFF_RQ};
    uint8_t *sVs[2] = {smem + Cfg::OFF_V, smem + Cfg::OFF_G};
    const uint32_t aPK = smem_addr(smem + Cfg::OFF_K);
    uint64_t *tma_b[2] = {tma_bar, tma_bar + 4};
    if (tid == 0) {
        mbar_init(tma_b[0], 1);
        mbar_init(tma_b[1], 1);
        mbar_init(mma_bar, 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 256);
    write_first<false>(sVs[0] + (DV / 16) * Cfg::BLK, tid, 1.f);
    write_first<false>(sVs[1] + (DV / 16) * Cfg::BLK, tid, 1.f);
#pragma unroll
    for (int f0 = F; f0 < Cfg::FT; f0 += 8) sts128(aPK + sw128_off(tid, f0), make_uint4(0u, 0u, 0u, 0u));
    __syncthreads();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane = (uint32_t)(warp * 32) << 16;
    // chunk c uses stage (c - c_begin) & 1; its loads go out when chunk c - 2's
    // MMA has finished with the stage, a whole chunk ahead of their use
    auto issue = [&](int chunk) {
        const int st = (chunk - c_begin) & 1, t0 = chunk * C;
        mbar_arrive_expect_tx(tma_b[st], Cfg::RAW + C * DV * 2);
        tma_load_3d(sKs[st], &tm_k, tma_b[st], 0, t0, bh);
        for (int x = 0; x < DV; x += 16) tma_load_3d(sVs[st] + (x / 16) * Cfg::BLK, &tm_v, tma_b[st], x, t0, bh);
    };
    int issued = c_begin, waited = c_begin;   // thread 0: chunks whose loads went out / were waited for
    if (tid == 0)
        for (; issued < c_end && issued < c_begin + 2; ++issued) issue(issued);
    uint32_t mph = 0;
    float *gL = reinterpret_cast<float *>(smem + Cfg::OFF_GATE);
    float seg_log = 0.f;   // gated: sum of the segment's gates
    for (int chunk = c_begin; chunk < c_end && !*abort_flag; ++chunk) {
        const int t0 = chunk * C, i = tid, st = (chunk - c_begin) & 1;
        const uint32_t aKs = smem_addr(sKs[st]), aV = smem_addr(sVs[st]);
        float Lrow = 0.f, Llast = 0.f;
        if constexpr (GATED) {
            Lrow = gate_prefix(p.logdecay + (size_t)bh * N + t0, i, min(C, N - t0), warp, tid & 31, true, gL, Llast);
            seg_log += Llast;
        }
        if (!mbar_wait(tma_b[st], (uint32_t)((chunk - c_begin) >> 1) & 1u)) *abort_flag = 1;
        waited = chunk + 1;
        {
            float x[16];
            raw_row16(aKs, i, x);
            tay_phi_row<0, 20>(aPK, i, x, t0 + i >= N, p);
        }
        if constexpr (GATED) {
            // S <- exp(L_last) S + sum_j exp(L_last - L_j) phi(k_j) [v_j | 1]^T
            const float w = __expf(Llast - Lrow);
            scale_row_sw32<false>(aV, i, 0, DV, w);
            write_first<false>(sVs[st] + (DV / 16) * Cfg::BLK, i, w);
            if (chunk > c_begin) decay_state_tiles<Cfg>(tmem, lane, warp, 0, NA, __expf(Llast));
        }
        full_sync();
        if (*abort_flag) break;
        if (tid == 0) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int m = Cfg::tile_m(t);
                const uint32_t a_base = aPK + (Cfg::tile_f0(t) / 64) * (C * 128);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + t * NA, smem_desc(a_base + kk * 2048, C * 128, 1024, kSw128),
                             smem_desc(aV + kk * 512, Cfg::BLK, 256, kSw32), idesc_bf16(m, NA, 1, 1),
                             chunk > c_begin || kk > 0);
            }
            mma_commit(mma_bar);
        }
        if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
        mph ^= 1u;
        if (tid == 0 && !*abort_flag && issued < c_end) issue(issued++);
        full_sync();
    }
    // after an early exit, let this block's own copies land (bounded)
    if (tid == 0 && *abort_flag)
        for (int c = waited; c < issued; ++c)
            mbar_wait(tma_b[(c - c_begin) & 1], (uint32_t)((c - c_begin) >> 1) & 1u, 100000000ull);
    if (!*abort_flag) {
        if (GATED && tid == 0) p.ws_log[(size_t)bh * p.P + seg] = seg_log;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (!state_quadrant<Cfg>(t, warp)) continue;
            const int f = state_row<Cfg>(t, warp, tid & 31);
            float *dst = p.ws_s + ((size_t)(bh * p.P + seg) * F + (f < 0 ? 0 : f)) * NA;
#pragma unroll 1
            for (int c0 = 0; c0 < NA; c0 += 16) {
                float v[16];
                tmem_ld16(tmem + t * NA + lane + c0, v);
                tmem_ld_wait();
                if (f >= 0)
#pragma unroll
                    for (int e = 0; e < 16; ++e) dst[c0 + e] = v[e];
            }
        }
    }
    full_sync();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// The elu state passes on a three-stage pipeline (256 threads).  Chunk k of a
// segment uses stage k % 3; the two threads of row r (r and r + 128) convert
// complementary parts of the row; once a chunk is converted one thread issues
// its MMA into the TMEM accumulator and the block goes on to the next chunk,
// whose conversion runs under that MMA.  Chunk k + 2's loads go out once the
// MMA of chunk k - 1 has released its stage.  Gated: the accumulator decays by
// the chunk's whole gate between two MMAs, so every thread waits for the
// previous chunk's MMA after converting and before decaying.
namespace bwd_detail {

// Columns [c_lo, c_hi) (multiples of 8) of row r of a bf16 SW32 tile of 128
// rows, rewritten as fp16 (times s with SCALE; without, the exact conversion).
template <bool SCALE>
__device__ __forceinline__ void row_to_f16(uint32_t tile, int r, int c_lo, int c_hi, float s)
{
#pragma unroll 1
    for (int c0 = c_lo; c0 < c_hi; c0 += 8) {
        const uint32_t a = tile + sw32_off(r, c0, 128);
        const uint4 u = lds128(a);
        if constexpr (SCALE) {
            float f[8];
            unpack8(u, f);
            sts128(a, make_uint4(pack_f16(f[0] * s, f[1] * s), pack_f16(f[2] * s, f[3] * s), pack_f16(f[4] * s, f[5] * s),
                                 pack_f16(f[6] * s, f[7] * s)));
        } else {
            sts128(a, make_uint4(bf16x2_to_f16x2(u.x), bf16x2_to_f16x2(u.y), bf16x2_to_f16x2(u.z), bf16x2_to_f16x2(u.w)));
        }
    }
}

// The accumulated increment (one state tile of NA columns in TMEM) to
// dst [F][NA]; this thread takes columns [c_lo, c_hi) of its lane's row.
template <class Cfg>
__device__ __forceinline__ void store_state_tile(float *dst, uint32_t t_lane, int wq, int l, int c_lo, int c_hi)
{
    if (!state_quadrant<Cfg>(0, wq)) return;
    const int f = state_row<Cfg>(0, wq, l);
    float *d = dst + (size_t)(f < 0 ? 0 : f) * Cfg::NA;
#pragma unroll 1
    for (int c0 = c_lo; c0 < c_hi; c0 += 16) {
        float v[16];
        tmem_ld16(t_lane + c0, v);
        tmem_ld_wait();
        if (f >= 0)
#pragma unroll
            for (int e = 0; e < 16; ++e) d[c0 + e] = v[e];
    }
}

}  // namespace bwd_detail

// S increments (elu): for each segment but the last, the sum over its tokens
// of phi(k_j) [v_j | 1]^T (gated: key j weighted by exp(L_last - L_j) within
// its chunk, the sum decayed by each later chunk's gate), fp16 operands like
// the forward-order pass that consumes them.
template <class Cfg, bool GATED = false>
__global__ void __launch_bounds__(256, 1)
bwd_sstate3_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const BwdParams p)
{
    using namespace bwd_detail;
    static_assert(!Cfg::TAYLOR, "elu shapes");
    constexpr int C = Cfg::C, D = Cfg::D, DV = Cfg::DV, NA = Cfg::NA;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *tma_b = reinterpret_cast<uint64_t *>(smem + Cfg::SP_BAR), *mma_b = tma_b + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_b + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tma_b + 7);
    float *gL = reinterpret_cast<float *>(smem + Cfg::SP_GATE);
    const int tid = threadIdx.x, warp = tid >> 5, wq = warp & 3, hh = warp >> 2, l = tid & 31;
    const int row = wq * 32 + l;
    const int bh = blockIdx.x / p.P, seg = blockIdx.x % p.P;
    if (seg == p.P - 1) return;   // the last segment's increment is never read
    const int c_begin = seg * p.cps, c_end = min(p.nchunks, c_begin + p.cps), n = c_end - c_begin;
    const int N = p.N;
    auto sA = [&](int st) { return smem + st * Cfg::SP_STAGE; };
    auto sB = [&](int st) { return smem + st * Cfg::SP_STAGE + Cfg::SP_A; };
    if (tid == 0) {
        for (int s2 = 0; s2 < 3; ++s2) {
            mbar_init(&tma_b[s2], 1);
            mbar_init(&mma_b[s2], 1);
        }
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 256);
    if (!GATED && hh == 0)
        for (int s2 = 0; s2 < 3; ++s2) write_first_f16(sB(s2) + (DV / 16) * Cfg::BLK, row, 1.f);
    full_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane = (uint32_t)(wq * 32) << 16;
    const int na_lo = hh ? Cfg::NA_SPLIT : 0, na_hi = hh ? NA : Cfg::NA_SPLIT;
    auto issue = [&](int k) {
        const int st = k % 3, t0 = (c_begin + k) * C;
        mbar_arrive_expect_tx(&tma_b[st], C * D * 2 + C * DV * 2);
        for (int x = 0; x < D; x += 64) tma_load_3d(sA(st) + (x / 64) * C * 128, &tm_k, &tma_b[st], x, t0, bh);
        for (int x = 0; x < DV; x += 16) tma_load_3d(sB(st) + (x / 16) * Cfg::BLK, &tm_v, &tma_b[st], x, t0, bh);
    };
    int issued = 0, waited = 0, mmas = 0;   // thread 0: chunks whose loads went out / were waited for / MMAs went out
    if (tid == 0)
        for (; issued < n && issued < 3; ++issued) issue(issued);
    float seg_log = 0.f;
    // every thread runs the same iterations and leaves only at the check after
    // the barrier, so a flag thread 0 sets after that check is seen by all at
    // the next one
    for (int k = 0; k < n; ++k) {
        const int st = k % 3, t0 = (c_begin + k) * C;
        const uint32_t aK = smem_addr(sA(st)), aV = smem_addr(sB(st));
        float Lrow = 0.f, Llast = 0.f;
        if constexpr (GATED) {
            Lrow = gate_prefix(p.logdecay + (size_t)bh * N + t0, row, min(C, N - t0), wq, l, hh == 0, gL, Llast);
            seg_log += Llast;
        }
        if (!mbar_wait(&tma_b[st], (uint32_t)(k / 3) & 1u)) *abort_flag = 1;
        if (tid == 0) waited = k + 1;
        const bool zero = t0 + row >= N;
        const float w = GATED ? __expf(Llast - Lrow) : 1.f;
        // phi(K) and V_aug in fp16: d = 128, the row's two threads take one
        // half of each; d = 64, one takes phi(K) and the other V_aug
        if (D == 128 || hh == 0) phi_block_f16(aK, row, zero, D == 128 ? hh : 0);
        if (D == 128 || hh == 1) {
            const int c_lo = D == 128 ? 64 * hh : 0, c_hi = D == 128 ? 64 * hh + 64 : DV;
            row_to_f16<GATED>(aV, row, c_lo, c_hi, w);
            if (GATED && c_lo == 0) write_first_f16(sB(st) + (DV / 16) * Cfg::BLK, row, w);
        }
        if constexpr (GATED) {
            if (k > 0) {
                if (!mbar_wait(&mma_b[(k - 1) % 3], (uint32_t)((k - 1) / 3) & 1u)) *abort_flag = 1;
                tc_fence_after();
                decay_state_tiles<Cfg>(tmem, lane, wq, na_lo, na_hi, __expf(Llast));
            }
        }
        full_sync();
        if (*abort_flag) break;
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                mma_bf16(tmem, smem_desc(aK + kk * 2048, C * 128, 1024, kSw128), smem_desc(aV + kk * 512, Cfg::BLK, 256, kSw32),
                         idesc_f16(Cfg::tile_m(0), NA, 1, 1), k > 0 || kk > 0);
            mma_commit(&mma_b[st]);
            mmas = k + 1;
            // the stage of chunk k - 1 takes chunk k + 2 once its MMA is done
            if (k >= 1 && issued < n) {
                if (mbar_wait(&mma_b[(k - 1) % 3], (uint32_t)((k - 1) / 3) & 1u)) issue(issued++);
                else *abort_flag = 1;
            }
        }
    }
    // thread 0: let its own copies land and its MMAs finish (bounded), then all read
    if (tid == 0) {
        for (int c = waited; c < issued; ++c) mbar_wait(&tma_b[c % 3], (uint32_t)(c / 3) & 1u, 100000000ull);
        if (mmas > 0 && !mbar_wait(&mma_b[(mmas - 1) % 3], (uint32_t)((mmas - 1) / 3) & 1u)) *abort_flag = 1;
        if (mmas < n) *abort_flag = 1;
    }
    full_sync();
    if (!*abort_flag) {
        if (GATED && tid == 0) p.ws_log[(size_t)bh * p.P + seg] = seg_log;
        store_state_tile<Cfg>(p.ws_s + (size_t)(bh * p.P + seg) * Cfg::F * NA, tmem + lane, wq, l, na_lo, na_hi);
    }
    full_sync();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// R increments (elu): for each segment but the first, the sum over its tokens
// of phi(q_i) G'_i^T (gated: chunks taken from the segment's end, query i
// weighted by exp(L_i), the sum decayed by each earlier chunk's gate), on the
// pipeline of bwd_sstate3_kernel with stages of [Q | dO_aug].
template <class Cfg, bool GATED = false>
__global__ void __launch_bounds__(256, 1)
bwd_rstate3_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                   const BwdParams p)
{
    using namespace bwd_detail;
    static_assert(!Cfg::TAYLOR, "elu shapes");
    constexpr int C = Cfg::C, D = Cfg::D, DV = Cfg::DV, NA = Cfg::NA;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *tma_b = reinterpret_cast<uint64_t *>(smem + Cfg::SP_BAR), *mma_b = tma_b + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_b + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tma_b + 7);
    float *gL = reinterpret_cast<float *>(smem + Cfg::SP_GATE);
    const int tid = threadIdx.x, warp = tid >> 5, wq = warp & 3, hh = warp >> 2, l = tid & 31;
    const int row = wq * 32 + l;
    const int bh = blockIdx.x / p.P, seg = blockIdx.x % p.P;
    if (seg == 0) return;   // the first segment's increment is never read
    const int c_begin = seg * p.cps, c_end = min(p.nchunks, c_begin + p.cps), n = c_end - c_begin;
    const int N = p.N;
    auto sA = [&](int st) { return smem + st * Cfg::SP_STAGE; };
    auto sB = [&](int st) { return smem + st * Cfg::SP_STAGE + Cfg::SP_A; };
    auto chunk_of = [&](int k) { return GATED ? c_end - 1 - k : c_begin + k; };
    if (tid == 0) {
        for (int s2 = 0; s2 < 3; ++s2) {
            mbar_init(&tma_b[s2], 1);
            mbar_init(&mma_b[s2], 1);
        }
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 256);
    full_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane = (uint32_t)(wq * 32) << 16;
    const int na_lo = hh ? Cfg::NA_SPLIT : 0, na_hi = hh ? NA : Cfg::NA_SPLIT;
    auto issue = [&](int k) {
        const int st = k % 3, t0 = chunk_of(k) * C;
        mbar_arrive_expect_tx(&tma_b[st], C * D * 2 + C * DV * 2);
        for (int x = 0; x < D; x += 64) tma_load_3d(sA(st) + (x / 64) * C * 128, &tm_q, &tma_b[st], x, t0, bh);
        for (int x = 0; x < DV; x += 16) tma_load_3d(sB(st) + (x / 16) * Cfg::BLK, &tm_do, &tma_b[st], x, t0, bh);
    };
    int issued = 0, waited = 0, mmas = 0;
    if (tid == 0)
        for (; issued < n && issued < 3; ++issued) issue(issued);
    for (int k = 0; k < n; ++k) {
        const int st = k % 3, t0 = chunk_of(k) * C;
        const bool valid = t0 + row < N;
        const uint32_t aQ = smem_addr(sA(st)), aG = smem_addr(sB(st));
        float Lrow = 0.f, Llast = 0.f;
        if constexpr (GATED)
            Lrow = gate_prefix(p.logdecay + (size_t)bh * N + t0, row, min(C, N - t0), wq, l, hh == 0, gL, Llast);
        // den_i, dden_i of this row (they do not depend on the loads)
        const float den = valid ? p.dd[((size_t)bh * N + t0 + row) * 2] : 1.f;
        const float dden = valid ? p.dd[((size_t)bh * N + t0 + row) * 2 + 1] : 0.f;
        if (!mbar_wait(&tma_b[st], (uint32_t)(k / 3) & 1u)) *abort_flag = 1;
        if (tid == 0) waited = k + 1;
        // phi(q_i) G'_i^T with G'_i = [dO_i / den_i | dden_i] (gated: times
        // exp(L_i)), taken as (phi(q_i) s_i) [dO_i | den_i dden_i]^T with
        // s_i = exp(L_i) / den_i: dO stays exact in bf16 and the scale rounds
        // once, with phi
        const float si = valid ? (GATED ? __expf(Lrow) : 1.f) / den : 0.f;
        if (D == 128 || hh == 0) phi_block_scaled<GATED>(aQ, row, si, D == 128 ? hh : 0);
        if ((D == 128 && hh == 0) || (D != 128 && hh == 1))
            write_dden(sB(st) + (DV / 16) * Cfg::BLK, row, valid ? den * dden : 0.f);
        if constexpr (GATED) {
            if (k > 0) {
                if (!mbar_wait(&mma_b[(k - 1) % 3], (uint32_t)((k - 1) / 3) & 1u)) *abort_flag = 1;
                tc_fence_after();
                decay_state_tiles<Cfg>(tmem, lane, wq, na_lo, na_hi, __expf(Llast));
            }
        }
        full_sync();
        if (*abort_flag) break;
        if (tid == 0) {
            // R_aug += phi(Q)^T G'   (M = the D features, N = NA, K = tokens)
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                mma_bf16(tmem, smem_desc(aQ + kk * 2048, C * 128, 1024, kSw128), smem_desc(aG + kk * 512, Cfg::BLK, 256, kSw32),
                         idesc_bf16(Cfg::tile_m(0), NA, 1, 1), k > 0 || kk > 0);
            mma_commit(&mma_b[st]);
            mmas = k + 1;
            if (k >= 1 && issued < n) {
                if (mbar_wait(&mma_b[(k - 1) % 3], (uint32_t)((k - 1) / 3) & 1u)) issue(issued++);
                else *abort_flag = 1;
            }
        }
    }
    if (tid == 0) {
        for (int c = waited; c < issued; ++c) mbar_wait(&tma_b[c % 3], (uint32_t)(c / 3) & 1u, 100000000ull);
        if (mmas > 0 && !mbar_wait(&mma_b[(mmas - 1) % 3], (uint32_t)((mmas - 1) / 3) & 1u)) *abort_flag = 1;
        if (mmas < n) *abort_flag = 1;
    }
    full_sync();
    if (!*abort_flag)
        store_state_tile<Cfg>(p.ws_r + (size_t)(bh * p.P + seg) * Cfg::F * NA, tmem + lane, wq, l, na_lo, na_hi);
    full_sync();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// R increments, Taylor map: for each segment but the first, sum over its
// tokens of phi(q_i) G'_i^T (needs den_i, dden_i from the forward-order pass);
// the pipeline of bwd_sstate_kernel with stages of [raw Q | G'_aug].
template <class Cfg, bool GATED = false>
__global__ void __launch_bounds__(128, 1)
bwd_rstate_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p)
{
    using namespace bwd_detail;
    static_assert(Cfg::TAYLOR, "the elu shapes take bwd_rstate3_kernel");
    constexpr int C = Cfg::C, DV = Cfg::DV, NA = Cfg::NA, F = Cfg::F, NT = Cfg::NT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *mma_bar = tma_bar + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_bar + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tma_bar + 3);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int bh = blockIdx.x / p.P, seg = blockIdx.x % p.P;
    if (seg == 0) return;   // the first segment's increment is never read
    const int c_begin = seg * p.cps, c_end = min(p.nchunks, c_begin + p.cps);
    const int N = p.N;
    // two stages of [raw Q | G'_aug], and one phi(Q) tile in the Q region
    uint8_t *sQs[2] = {smem + Cfg::OFF_RQ, smem + Cfg::OFF_RK};
    uint8_t *sGs[2] = {smem + Cfg::OFF_G, smem + Cfg::OFF_V};
    const uint32_t aPQ = smem_addr(smem + Cfg::OFF_Q);
    uint64_t *tma_b[2] = {tma_bar, tma_bar + 4};
    if (tid == 0) {
        mbar_init(tma_b[0], 1);
        mbar_init(tma_b[1], 1);
        mbar_init(mma_bar, 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 256);
#pragma unroll
    for (int f0 = F; f0 < Cfg::FT; f0 += 8) sts128(aPQ + sw128_off(tid, f0), make_uint4(0u, 0u, 0u, 0u));
    __syncthreads();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane = (uint32_t)(warp * 32) << 16;
    // The it-th chunk taken (forward order; gated: from the segment's end, so
    // that R can decay as it goes) uses stage it & 1; its loads go out when
    // the (it - 2)-th chunk's MMA has finished with the stage.
    const int nch = c_end - c_begin;
    auto chunk_of = [&](int it) { return GATED ? c_end - 1 - it : c_begin + it; };
    auto issue = [&](int it) {
        const int st = it & 1, t0 = chunk_of(it) * C;
        mbar_arrive_expect_tx(tma_b[st], Cfg::RAW + C * DV * 2);
        tma_load_3d(sQs[st], &tm_q, tma_b[st], 0, t0, bh);
        for (int x = 0; x < DV; x += 16) tma_load_3d(sGs[st] + (x / 16) * Cfg::BLK, &tm_do, tma_b[st], x, t0, bh);
    };
    int issued = 0, waited = 0;   // counts of chunks taken
    if (tid == 0)
        for (; issued < nch && issued < 2; ++issued) issue(issued);
    uint32_t mph = 0;
    float *gL = reinterpret_cast<float *>(smem + Cfg::OFF_GATE);
    for (int it = 0; it < nch && !*abort_flag; ++it) {
        const int chunk = chunk_of(it);
        const int t0 = chunk * C, i = tid, st = it & 1;
        const bool valid = t0 + i < N;
        uint8_t *sG = sGs[st];
        const uint32_t aQs = smem_addr(sQs[st]), aG = smem_addr(sG);
        float Lrow = 0.f, Llast = 0.f;
        if constexpr (GATED)
            Lrow = gate_prefix(p.logdecay + (size_t)bh * N + t0, i, min(C, N - t0), warp, tid & 31, true, gL, Llast);
        if (!mbar_wait(tma_b[st], (uint32_t)(it >> 1) & 1u)) *abort_flag = 1;
        waited = it + 1;
        {
            float x[16];
            raw_row16(aQs, i, x);
            tay_phi_row<0, 20>(aPQ, i, x, false, p);
        }
        {
            // gated: query row i enters R scaled by exp(L_i)
            const float e = GATED ? __expf(Lrow) : 1.f;
            const float den = valid ? p.dd[((size_t)bh * N + t0 + i) * 2] : 1.f;
            const float dden = valid ? e * p.dd[((size_t)bh * N + t0 + i) * 2 + 1] : 0.f;
            const float inv = valid ? e / den : 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < DV; c0 += 8) {
                float go[8];
                const uint32_t a = aG + sw32_off(i, c0, C);
                unpack8(lds128(a), go);
                sts128(a, make_uint4(pack_bf16(go[0] * inv, go[1] * inv), pack_bf16(go[2] * inv, go[3] * inv),
                                     pack_bf16(go[4] * inv, go[5] * inv), pack_bf16(go[6] * inv, go[7] * inv)));
            }
            write_dden(sG + (DV / 16) * Cfg::BLK, i, dden);
        }
        // gated: R <- exp(L_last) R + sum_i exp(L_i) phi(q_i) G'_i^T
        if (GATED && it > 0) decay_state_tiles<Cfg>(tmem, lane, warp, 0, NA, __expf(Llast));
        full_sync();
        if (*abort_flag) break;
        if (tid == 0) {
            // R_aug += phi(Q)^T G'   (M = F features, N = NA, K = tokens)
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int m = Cfg::tile_m(t);
                const uint32_t a_base = aPQ + (Cfg::tile_f0(t) / 64) * (C * 128);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + t * NA, smem_desc(a_base + kk * 2048, C * 128, 1024, kSw128),
                             smem_desc(aG + kk * 512, Cfg::BLK, 256, kSw32), idesc_bf16(m, NA, 1, 1),
                             it > 0 || kk > 0);
            }
            mma_commit(mma_bar);
        }
        if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
        mph ^= 1u;
        if (tid == 0 && !*abort_flag && issued < nch) issue(issued++);
        full_sync();
    }
    if (tid == 0 && *abort_flag)
        for (int c = waited; c < issued; ++c) mbar_wait(tma_b[c & 1], (uint32_t)(c >> 1) & 1u, 100000000ull);
    if (!*abort_flag) {
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (!state_quadrant<Cfg>(t, warp)) continue;
            const int f = state_row<Cfg>(t, warp, tid & 31);
            float *dst = p.ws_r + ((size_t)(bh * p.P + seg) * F + (f < 0 ? 0 : f)) * NA;
#pragma unroll 1
            for (int c0 = 0; c0 < NA; c0 += 16) {
                float v[16];
                tmem_ld16(tmem + t * NA + lane + c0, v);
                tmem_ld_wait();
                if (f >= 0)
#pragma unroll
                    for (int e = 0; e < 16; ++e) dst[c0 + e] = v[e];
            }
        }
    }
    full_sync();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// Reverse-order pass: dk and dv.  256 threads: warps w and w + 4 share the
// TMEM lanes of rows 32 (w % 4) .. + 31, and every per-row step is split
// between them by columns (the first half of the columns to warps 0-3).
template <class Cfg, bool GATED = false>
__global__ void __launch_bounds__(256, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                const BwdParams p)
{
    using namespace bwd_detail;
    constexpr int C = Cfg::C, D = Cfg::D, DV = Cfg::DV, NA = Cfg::NA, F = Cfg::F, NT = Cfg::NT;
    constexpr bool TAY = Cfg::TAYLOR;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *mma_bar = tma_bar + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_bar + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tma_bar + 3);
    const int tid = threadIdx.x, warp = tid >> 5, wq = warp & 3, hh = warp >> 2, l = tid & 31;
    const int row = wq * 32 + l;   // this thread's token row / TMEM lane
    float *red = reinterpret_cast<float *>(smem + Cfg::OFF_RED);
    const int bh = blockIdx.x / p.P, seg = blockIdx.x % p.P;
    const int c_begin = seg * p.cps, c_end = min(p.nchunks, c_begin + p.cps);
    const int N = p.N;
    uint8_t *sQ = smem + Cfg::OFF_Q, *sK = smem + Cfg::OFF_K, *sV = smem + Cfg::OFF_V, *sG = smem + Cfg::OFF_G,
            *sR = smem + Cfg::OFF_S, *sGL = smem + Cfg::OFF_SL;   // G' bf16 remainder
    const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV), aG = smem_addr(sG), aR = smem_addr(sR),
                   aGL = smem_addr(sGL), aRQ = smem_addr(smem + Cfg::OFF_RQ), aRK = smem_addr(smem + Cfg::OFF_RK);
    if (tid == 0) {
        mbar_init(tma_bar, 1);
        mbar_init(mma_bar, 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 0) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    if (hh == 0) write_ones_block(sV + (DV / 16) * Cfg::BLK, row);
    if constexpr (TAY) {
#pragma unroll
        for (int f0 = F; f0 < Cfg::FT; f0 += 8)
            sts128((hh ? aK : aQ) + sw128_off(row, f0), make_uint4(0u, 0u, 0u, 0u));
    }
    __syncthreads();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane = (uint32_t)(wq * 32) << 16;
    const int na_lo = hh ? Cfg::NA_SPLIT : 0, na_hi = hh ? NA : Cfg::NA_SPLIT;   // this thread's columns of R_aug
    const uint32_t tA = tmem, tX = tmem + Cfg::COL_X, tR = tmem + Cfg::COL_R, tPL = tmem + Cfg::COL_PL;
    float *gL = reinterpret_cast<float *>(smem + Cfg::OFF_GATE);   // gated: the chunk's prefix sums of the gates
    float *dr = gL + C + 8;   // gated: r - bf16(r) per feature, r = R's normaliser column
    auto snap_r = [&](int f, int c0, const float *v) {
        sts128(aR + sw32_off(f, c0, F), make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                                   pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7])));
        sts128(aR + sw32_off(f, c0 + 8, F), make_uint4(pack_bf16(v[8], v[9]), pack_bf16(v[10], v[11]),
                                                       pack_bf16(v[12], v[13]), pack_bf16(v[14], v[15])));
        if (GATED && c0 == DV) dr[f] = v[0] - bf16_round(v[0]);
    };

    // ---- R entering the segment: sum of the later segments' increments
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        if (!state_quadrant<Cfg>(t, wq)) continue;
        const int f = state_row<Cfg>(t, wq, l);
        for (int c0 = na_lo; c0 < na_hi; c0 += 16) {
            float v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0.f;
            if (f >= 0) {
                if constexpr (GATED) {
                    // R seen from the end of segment s2 - 1 is s2's increment plus
                    // R at s2's end decayed by s2's gates; from the last segment down
                    for (int s2 = p.P - 1; s2 > seg; --s2) {
                        const float *src = p.ws_r + ((size_t)(bh * p.P + s2) * F + f) * NA + c0;
                        const float d = s2 == p.P - 1 ? 0.f : __expf(p.ws_log[(size_t)bh * p.P + s2]);
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = fmaf(v[e], d, src[e]);
                    }
                } else {
                    for (int s2 = seg + 1; s2 < p.P; ++s2) {
                        const float *src = p.ws_r + ((size_t)(bh * p.P + s2) * F + f) * NA + c0;
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] += src[e];
                    }
                }
            }
            tmem_st16(tR + t * NA + lane + c0, v);
            if (f >= 0) snap_r(f, c0, v);
        }
    }
    tmem_st_wait();
    full_sync();

    uint32_t tph = 0, mph = 0;
    for (int chunk = c_end - 1; chunk >= c_begin && !*abort_flag; --chunk) {
        const int t0 = chunk * C, j = row;
        const bool valid = t0 + j < N;
        if (tid == 0) {
            // the previous chunk's dk left from the K tile (its raw tile for Taylor)
            if (chunk < c_end - 1) bulk_wait_read();
            mbar_arrive_expect_tx(tma_bar, TAY ? 2 * Cfg::RAW + 2 * C * DV * 2 : 2 * C * D * 2 + 2 * C * DV * 2);
            if constexpr (TAY) {
                tma_load_3d(smem + Cfg::OFF_RQ, &tm_q, tma_bar, 0, t0, bh);
                tma_load_3d(smem + Cfg::OFF_RK, &tm_k, tma_bar, 0, t0, bh);
            } else {
                for (int x = 0; x < D; x += 64) {
                    tma_load_3d(sQ + (x / 64) * C * 128, &tm_q, tma_bar, x, t0, bh);
                    tma_load_3d(sK + (x / 64) * C * 128, &tm_k, tma_bar, x, t0, bh);
                }
            }
            for (int x = 0; x < DV; x += 16) {
                tma_load_3d(sV + (x / 16) * Cfg::BLK, &tm_v, tma_bar, x, t0, bh);
                tma_load_3d(sG + (x / 16) * Cfg::BLK, &tm_do, tma_bar, x, t0, bh);
            }
        }
        if (!mbar_wait(tma_bar, tph)) *abort_flag = 1;
        tph ^= 1u;
        // gated: L over the chunk; exp(L_i - L_j) weights pair (i, j),
        // exp(L_last - L_j) the later chunks' terms of key j, exp(L_i) query i's
        // term of the R update
        float Lrow = 0.f, Llast = 0.f;
        if constexpr (GATED)
            Lrow = gate_prefix(p.logdecay + (size_t)bh * N + t0, row, min(C, N - t0), wq, l, hh == 0, gL, Llast);
        if constexpr (TAY) {
            float xq[16], xk[16];
            raw_row16(aRQ, j, xq);
            raw_row16(aRK, j, xk);
            if (hh == 0) {
                tay_phi_row<0, 10>(aQ, j, xq, false, p);
                tay_phi_row<0, 10>(aK, j, xk, !valid, p);
            } else {
                tay_phi_row<80, 10>(aQ, j, xq, false, p);
                tay_phi_row<80, 10>(aK, j, xk, !valid, p);
            }
        } else if (D == 128) {
            phi_block_inplace<GATED>(aQ, j, false, hh);
            phi_block_inplace<GATED>(aK, j, !valid, hh);
        } else if (hh == 0) {
            phi_block_inplace<GATED>(aQ, j, false, 0);
        } else {
            phi_block_inplace<GATED>(aK, j, !valid, 0);
        }
        float dden_row;
        {
            // G' row j (this thread's token as a query): [dO/den | dden] as bf16
            // plus its bf16 remainder (dA^T below uses both)
            const float den = valid ? p.dd[((size_t)bh * N + t0 + j) * 2] : 1.f;
            dden_row = valid ? p.dd[((size_t)bh * N + t0 + j) * 2 + 1] : 0.f;
            const float dden = dden_row;
            const float inv = valid ? 1.f / den : 0.f;
#pragma unroll 1
            for (int c0 = hh * (DV / 2); c0 < (hh + 1) * (DV / 2); c0 += 8) {
                float go[8];
                const uint32_t a = aG + sw32_off(j, c0, C);
                unpack8(lds128(a), go);
#pragma unroll
                for (int e = 0; e < 8; ++e) go[e] *= inv;
                sts128(a, make_uint4(pack_bf16(go[0], go[1]), pack_bf16(go[2], go[3]), pack_bf16(go[4], go[5]),
                                     pack_bf16(go[6], go[7])));
                float r[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) r[e] = go[e] - __bfloat162float(__float2bfloat16_rn(go[e]));
                sts128(aGL + sw32_off(j, c0, C), make_uint4(pack_bf16(r[0], r[1]), pack_bf16(r[2], r[3]),
                                                            pack_bf16(r[4], r[5]), pack_bf16(r[6], r[7])));
            }
            if (hh == 0) {
                write_dden(sG + (DV / 16) * Cfg::BLK, j, dden);
                write_dden(sGL + (DV / 16) * Cfg::BLK, j, dden - __bfloat162float(__float2bfloat16_rn(dden)));
            }
        }
        full_sync();
        if (*abort_flag) break;

        // A^T = phi(K) phi(Q)^T (Taylor: raw K Q^T) ;  dA^T = V_aug G'^T
        if (tid == 0) {
            if constexpr (TAY) {
                mma_bf16(tA, smem_desc(aRK, 16, 256, kSw32), smem_desc(aRQ, 16, 256, kSw32), idesc_bf16(128, 128, 0, 0),
                         false);
            } else {
#pragma unroll
                for (int kk = 0; kk < F / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (C * 128) + (kk & 3) * 32;
                    mma_bf16(tA, smem_desc(aK + off, 16, 1024, kSw128), smem_desc(aQ + off, 16, 1024, kSw128),
                             idesc_bf16(128, 128, 0, 0), kk > 0);
                }
            }
#pragma unroll
            for (int kk = 0; kk < NA / 16; ++kk) {
                mma_bf16(tX, smem_desc(aV + kk * Cfg::BLK, 16, 256, kSw32), smem_desc(aG + kk * Cfg::BLK, 16, 256, kSw32),
                         idesc_bf16(128, 128, 0, 0), kk > 0);
                mma_bf16(tX, smem_desc(aV + kk * Cfg::BLK, 16, 256, kSw32), smem_desc(aGL + kk * Cfg::BLK, 16, 256, kSw32),
                         idesc_bf16(128, 128, 0, 0), true);
            }
            mma_commit(mma_bar);
        }
        if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
        mph ^= 1u;
        tc_fence_after();
        // row j keeps the queries i >= j
        float c_part = 0.f;   // gated: this thread's part of c_j = sum_i dL/dw_ij w_ij
        if constexpr (GATED) {
            c_part = mask_pack_both_gate<TAY>(tA + lane, tX + lane, tPL + lane, 64 * hh, p.inv_c3, p.k2, Lrow, gL,
                                              red + wq * C, [&](int i) { return i >= j; });
        } else {
            mask_pack_half_g<false, TAY>(tA + lane, tA + lane, 64 * hh, true, p.inv_c3, p.k2,
                                         [&](int i) { return i >= j; });
            mask_pack_half_hilo(tX + lane, tA + lane + 64, tPL + lane, 64 * hh, [&](int i) { return i >= j; });
        }
        full_sync();
        // gated: r_j's part over this chunk's keys (token j as a query), from the
        // four quadrants' column sums
        const float r_chunk = GATED ? red[j] + red[C + j] + red[2 * C + j] + red[3 * C + j] : 0.f;
        if constexpr (GATED) {
            // the later chunks' term of dV first, scaled per key row by exp(L_last - L_j)
            if (tid == 0) {
                const uint32_t id = idesc_bf16(128, DV, 0, 1);
#pragma unroll
                for (int kk = 0; kk < F / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (C * 128) + (kk & 3) * 32;
                    mma_bf16(tX, smem_desc(aK + off, 16, 1024, kSw128), smem_desc(aR + kk * 512, Cfg::S_BLK, 256, kSw32),
                             id, kk > 0);
                }
                mma_commit(mma_bar);
            }
            if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
            mph ^= 1u;
            tc_fence_after();
            tmem_scale(tX + lane, hh * (DV / 2), (hh + 1) * (DV / 2), __expf(Llast - Lrow));
            full_sync();
        }

        // dV = P^T G + phi(K) R
        if (tid == 0) {
            const uint32_t id = idesc_bf16(128, DV, 0, 1);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                mma_bf16_ts(tX, tA + kk * 8, smem_desc(aG + kk * 512, Cfg::BLK, 256, kSw32), id, GATED || kk > 0);
#pragma unroll
            for (int kk = 0; kk < (GATED ? 0 : F / 16); ++kk) {
                const uint32_t off = (kk >> 2) * (C * 128) + (kk & 3) * 32;
                mma_bf16(tX, smem_desc(aK + off, 16, 1024, kSw128), smem_desc(aR + kk * 512, Cfg::S_BLK, 256, kSw32),
                         id, true);
            }
            mma_commit(mma_bar);
        }
        if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
        mph ^= 1u;
        tc_fence_after();
        {
            // ungated: dv goes as SW128 rows to the G' remainder tile (read only by
            // dA^T above) and leaves by TMA with dk; gated: row stores (that tile
            // still feeds the R update)
            __nv_bfloat16 *dvrow = reinterpret_cast<__nv_bfloat16 *>(p.dv) + ((size_t)bh * N + t0 + j) * DV;
#pragma unroll 1
            for (int c0 = hh * (DV / 2); c0 < (hh + 1) * (DV / 2); c0 += 16) {
                float g[16];
                tmem_ld16(tX + lane + c0, g);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; e += 8) {
                    const uint4 u = make_uint4(pack_bf16(g[e], g[e + 1]), pack_bf16(g[e + 2], g[e + 3]),
                                               pack_bf16(g[e + 4], g[e + 5]), pack_bf16(g[e + 6], g[e + 7]));
                    if constexpr (GATED) {
                        if (valid) *reinterpret_cast<uint4 *>(dvrow + c0 + e) = u;
                    } else {
                        sts128(aGL + sw128_off(j, c0 + e), u);
                    }
                }
            }
        }
        if constexpr (GATED) {
            // G''s last use below is the R update: scale query row j by exp(L_j)
            // (head and remainder: dL/dg sums phi(k) . dphi(k) over the sequence,
            // and a bf16 G' in R leaves ~2^-9 of noise in each of those terms),
            // and decay R by the chunk's whole gate
            const float e = __expf(Lrow);
            scale_row_hilo(aG, aGL, j, hh * (DV / 2), (hh + 1) * (DV / 2), e);
            if (hh == 0) {
                const float x = dden_row * e;
                write_dden(sG + (DV / 16) * Cfg::BLK, j, x);
                write_dden(sGL + (DV / 16) * Cfg::BLK, j, x - bf16_round(x));
            }
            decay_state_tiles<Cfg>(tR, lane, wq, na_lo, na_hi, __expf(Llast));
        }
        full_sync();
        if constexpr (GATED) {
            // the later chunks' term of dphi(K) first, scaled per key row by exp(L_last - L_j)
            if (tid == 0) {
#pragma unroll
                for (int kk = 0; kk < NA / 16; ++kk)
                    mma_bf16(tX, smem_desc(aV + kk * Cfg::BLK, 16, 256, kSw32),
                             smem_desc(aR + kk * Cfg::S_BLK, 16, 256, kSw32), idesc_bf16(128, F, 0, 0), kk > 0);
                mma_commit(mma_bar);
            }
            if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
            mph ^= 1u;
            tc_fence_after();
            // the later chunks' part of c_j: phi(k_j) . (their term of dphi(k_j))
            const float w = __expf(Llast - Lrow);
            float dot;
            if constexpr (TAY) {
                float xk[16];
                raw_row16(aRK, j, xk);
                dot = hh == 0 ? tay_dot_half<true, 0>(tX + lane, xk, dr, p) : tay_dot_half<true, 1>(tX + lane, xk, dr, p);
            } else {
                dot = elu_dot_cols<false, true>(tX + lane, aK, j, hh * (F / 2), (hh + 1) * (F / 2), dr);
            }
            c_part = fmaf(w, dot, c_part);
            tmem_scale(tX + lane, hh * (F / 2), (hh + 1) * (F / 2), w);
            full_sync();
        }

        // dphi(K) = dP^T phi(Q) + V_aug R_aug^T ;  then R_aug += phi(Q)^T G'
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                mma_bf16_ts(tX, tA + 64 + kk * 8, smem_desc(aQ + kk * 2048, C * 128, 1024, kSw128),
                            idesc_bf16(128, F, 0, 1), GATED || kk > 0);
                mma_bf16_ts(tX, tPL + kk * 8, smem_desc(aQ + kk * 2048, C * 128, 1024, kSw128),
                            idesc_bf16(128, F, 0, 1), true);
            }
#pragma unroll
            for (int kk = 0; kk < (GATED ? 0 : NA / 16); ++kk)
                mma_bf16(tX, smem_desc(aV + kk * Cfg::BLK, 16, 256, kSw32), smem_desc(aR + kk * Cfg::S_BLK, 16, 256, kSw32),
                         idesc_bf16(128, F, 0, 0), true);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int m = Cfg::tile_m(t);
                const uint32_t a_base = aQ + (Cfg::tile_f0(t) / 64) * (C * 128);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {
                    mma_bf16(tR + t * NA, smem_desc(a_base + kk * 2048, C * 128, 1024, kSw128),
                             smem_desc(aG + kk * 512, Cfg::BLK, 256, kSw32), idesc_bf16(m, NA, 1, 1), true);
                    if constexpr (GATED)
                        mma_bf16(tR + t * NA, smem_desc(a_base + kk * 2048, C * 128, 1024, kSw128),
                                 smem_desc(aGL + kk * 512, Cfg::BLK, 256, kSw32), idesc_bf16(m, NA, 1, 1), true);
                }
            }
            mma_commit(mma_bar);
        }
        if (!mbar_wait(mma_bar, mph)) *abort_flag = 1;
        mph ^= 1u;
        tc_fence_after();
        {
            if constexpr (TAY) {
                float x[16], dx[16], sd = 0.f;
                raw_row16(aRK, j, x);
#pragma unroll
                for (int c = 0; c < 16; ++c) dx[c] = 0.f;
                if (hh == 0) tay_vjp_half<0>(tX + lane, x, dx, sd, p);
                else tay_vjp_half<1>(tX + lane, x, dx, sd, p);
                float d8[8], sd_all;
                tay_combine(red + 6 * C, red + 2 * C, hh, j, dx, sd, d8, sd_all);
                // dk over its own raw k (read by both threads of the row before the
                // barrier in tay_combine); one TMA store per chunk
                sts128(aRK + sw32_off(j, 8 * hh, 128), make_uint4(pack_bf16(d8[0], d8[1]), pack_bf16(d8[2], d8[3]),
                                                                  pack_bf16(d8[4], d8[5]), pack_bf16(d8[6], d8[7])));
            } else {
#pragma unroll 1
                for (int c0 = hh * (F / 2); c0 < (hh + 1) * (F / 2); c0 += 16) {
                    float g[16], ph[16];
                    tmem_ld16(tX + lane + c0, g);
                    tmem_ld_wait();
                    unpack8(lds128(aK + sw128_off(j, c0)), ph);
                    unpack8(lds128(aK + sw128_off(j, c0 + 8)), ph + 8);
                    // dk over the thread's own phi(k) entries (same SW128 layout)
#pragma unroll
                    for (int e = 0; e < 16; e += 8)
                        sts128(aK + sw128_off(j, c0 + e), make_uint4(
                            pack_bf16(g[e] * fminf(ph[e], 1.f), g[e + 1] * fminf(ph[e + 1], 1.f)),
                            pack_bf16(g[e + 2] * fminf(ph[e + 2], 1.f), g[e + 3] * fminf(ph[e + 3], 1.f)),
                            pack_bf16(g[e + 4] * fminf(ph[e + 4], 1.f), g[e + 5] * fminf(ph[e + 5], 1.f)),
                            pack_bf16(g[e + 6] * fminf(ph[e + 6], 1.f), g[e + 7] * fminf(ph[e + 7], 1.f))));
                }
            }
            if constexpr (GATED) {
                // c_j - r_j: c_j = phi(k_j) . dphi(k_j) summed over the row's two
                // threads; r_j = the chunk's part above plus the earlier chunks'
                // part the forward-order pass left in cvec
                red[4 * C + hh * C + j] = c_part;
                __syncthreads();
                if (hh == 0 && valid) {
                    float *cj = p.cvec + (size_t)bh * N + t0 + j;
                    *cj = red[4 * C + j] + red[5 * C + j] - r_chunk - *cj;
                }
            }
            if (chunk > c_begin) {
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    if (!state_quadrant<Cfg>(t, wq)) continue;
                    const int f = state_row<Cfg>(t, wq, l);
#pragma unroll 1
                    for (int c0 = na_lo; c0 < na_hi; c0 += 16) {
                        float v[16];
                        tmem_ld16(tR + t * NA + lane + c0, v);
                        tmem_ld_wait();
                        if (f >= 0) snap_r(f, c0, v);
                    }
                }
            }
        }
        full_sync();
        // the chunk's dk (and, ungated, dv) leave by TMA (rows past the slice's
        // end clipped)
        if (tid == 0 && !*abort_flag) {
            if constexpr (TAY) tma_store_3d(&tm_dk, smem + Cfg::OFF_RK, 0, t0, bh);
            else
                for (int x = 0; x < D; x += 64) tma_store_3d(&tm_dk, sK + (x / 64) * C * 128, x, t0, bh);
            if constexpr (!GATED)
                for (int x = 0; x < DV; x += 64) tma_store_3d(&tm_dv, sGL + (x / 64) * C * 128, x, t0, bh);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait_all();
    full_sync();
    if (warp == 0) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}


// ---------------------------------------------------------------------------
// Gated form: dL/dg_l = - sum_{m >= l} x_m per head, x_m = c_m - r_m from the
// two passes.  g_l scales every weight w_ij with j < l <= i, so dL/dg_l is the
// sum of M_ij = dL/dw_ij w_ij over those pairs; with r_m = sum_j M_mj (a row)
// and c_m = sum_i M_im (a column), sum_{m >= l} (r_m - c_m) is exactly that sum
// for any M.  (In exact arithmetic r_m = 0, the weights of a query entering y_m
// as a ratio; the kernels' own r_m is kept because their c_m and r_m then come
// from the same rounded pair terms for the pairs inside a chunk.)
// One block per head walks the sequence from its end in tiles of 1024.
__global__ void __launch_bounds__(1024, 1) bwd_dg_kernel(const float *c, float *dg, int N)
{
    __shared__ float wsum[32];
    const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float *cb = c + (size_t)bh * N;
    float *db = dg + (size_t)bh * N;
    float carry = 0.f;   // sum of c after the current tile
    for (int end = N; end > 0; end -= 1024) {
        const int idx = end - 1 - tid;   // thread t: position end-1-t
        float x = idx >= 0 ? cb[idx] : 0.f;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        float before = 0.f, total = 0.f;
        for (int w2 = 0; w2 < 32; ++w2) {
            const float t = wsum[w2];
            if (w2 < warp) before += t;
            total += t;
        }
        // position 0: no pair j < 0 <= i exists, so dL/dg_0 is zero by
        // definition (the suffix sum is zero only up to rounding)
        if (idx >= 0) db[idx] = idx == 0 ? 0.f : -(carry + before + x);
        carry += total;
        __syncthreads();
    }
}

}  // namespace la
