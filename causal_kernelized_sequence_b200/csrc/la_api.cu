// la_api.cu -- the C ABI of libla (declared in include/la.h): argument
// validation, kernel selection and launch.  The library is one translation
// unit: the kernel headers below are included here.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <atomic>
#include <utility>
#include <mutex>

#include "../../include/la.h"
#include <cstdio>
#include <utility>

#include "la_device.cuh"
#include "la_simt.cuh"
#include "la_decode.cuh"
#include "la_prefill_sm100.cuh"
#include "la_bwd_sm100.cuh"
#include "la_fwd_split_sm100.cuh"
#include "la_swa.cuh"

using namespace la;

namespace {

constexpr size_t kSmemLimit = 227 * 1024;

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

bool valid_enums(int fmap, int dtype)
{
    return (fmap == LA_FMAP_ELU1 || fmap == LA_FMAP_TAYLOR2 || fmap == LA_FMAP_TAYLOR2_SYM) &&
           (dtype == LA_F32 || dtype == LA_BF16);
}

// Sizes this build supports (valid but unsupported -> LA_ERR_UNSUPPORTED).
bool supported_dims(int fmap, int dqk, int dv)
{
    if (dv < 1 || dv > 128) return false;
    if (fmap == LA_FMAP_ELU1) return dqk >= 1 && dqk <= 128;
    return dqk >= 1 && dqk <= 16;
}

FmapParams make_fmap(int fmap, int dqk)
{
    FmapParams p;
    p.fmap = fmap;
    p.dqk = dqk;
    p.F = (int)la_feature_dim(fmap, dqk);
    p.inv_c1 = (float)(1.0 / pow((double)dqk, 0.25));
    p.inv_c2 = (float)(1.0 / (sqrt(2.0) * sqrt((double)dqk)));
    p.inv_c3 = (float)(1.0 / sqrt((double)dqk));
    return p;
}

// Common shape checks; returns LA_OK or the error to report.
la_status check_shape(int B, int H, int N, int dqk, int dv, int fmap, int dtype)
{
    if (!valid_enums(fmap, dtype)) return LA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || N < 1 || dqk < 1 || dv < 1) return LA_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)B * H * N;
    const int64_t widest = dqk > dv ? dqk : dv;
    if (rows * widest >= ((int64_t)1 << 31)) return LA_ERR_INVALID_ARG;
    if (!supported_dims(fmap, dqk, dv)) return LA_ERR_UNSUPPORTED;
    const int64_t F = la_feature_dim(fmap, dqk);
    if ((int64_t)B * H * F * dv >= ((int64_t)1 << 31)) return LA_ERR_INVALID_ARG;
    return LA_OK;
}

// The kernels run on the calling thread's current device and dereference
// the pointers they are given there.  A first operand that lives on another
// device, or in host memory the device cannot address, is refused before any
// launch (a launch would read another device's addresses through this one's
// page tables).  Device memory of the current device and managed memory pass.
la_status check_on_current_device(const void *p)
{
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        (void)cudaGetLastError();   // the query's error is the caller's argument, not a sticky state
        return LA_ERR_INVALID_ARG;
    }
    if (a.type == cudaMemoryTypeManaged) return LA_OK;
    if (a.type != cudaMemoryTypeDevice) return LA_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return LA_ERR_CUDA;
    return a.device == dev ? LA_OK : LA_ERR_INVALID_ARG;
}

la_status launch_status()
{
    const cudaError_t e = cudaGetLastError();
#ifdef LA_DEBUG_LAUNCH
    if (e != cudaSuccess) fprintf(stderr, "libla launch error: %s\n", cudaGetErrorString(e));
#endif
    return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

// Launch as a programmatic dependent of the previous kernel in the stream:
// the grid may be scheduled onto SMs that kernel has left once all its blocks
// have started (every tensor-core forward kernel triggers at its start), and
// each of these kernels waits for the previous one to complete (its writes
// visible) before it touches global memory.
template <typename... KArgs, typename... Args>
la_status launch_pdl(void (*kernel)(KArgs...), int grid, int threads, int smem, cudaStream_t stream, Args &&...args)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e == cudaSuccess) return LA_OK;
#ifdef LA_DEBUG_LAUNCH
    fprintf(stderr, "libla launch error: %s\n", cudaGetErrorString(e));
#endif
    (void)cudaGetLastError();   // consume it, as launch_status does for the other launches
    return LA_ERR_CUDA;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device) and
// size; later calls (for example during CUDA-graph capture) make no API call.
// The table is atomic because calls may come from several host threads; two
// threads racing on a first call both set the same attribute, which is harmless.
template <auto kernel>
la_status set_smem(size_t bytes)
{
    if (bytes <= 48 * 1024) return LA_OK;
    static std::atomic<size_t> done[64];  // one table per kernel, zero-initialised
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LA_ERR_CUDA;
    if (done[dev].load(std::memory_order_acquire) >= bytes) return LA_OK;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return LA_ERR_CUDA;
    done[dev].store(bytes, std::memory_order_release);
    return LA_OK;
}

// Kernel selection, shared by the entry points and la_kernel_plan.
enum class Path { Invalid, FwdSimt, FwdSplit, FwdTc, BwdSimt, BwdTc, DecodeSimt, DecodeVec };

// Shapes with a tensor-core forward: bf16 I/O and (elu, dqk = dv in {64,128})
// or (either Taylor map, dqk = 16, dv = 64).
bool tc_forward_shape(int dqk, int dv, int fmap, int dtype)
{
    if (dtype != LA_BF16) return false;
    if (fmap == LA_FMAP_ELU1) return dqk == dv && (dqk == 64 || dqk == 128);
    return dqk == 16 && dv == 64;
}

Path select_forward(int B, int H, int N, int dqk, int dv, int fmap, int dtype)
{
    if (check_shape(B, H, N, dqk, dv, fmap, dtype) != LA_OK) return Path::Invalid;
    if (dtype == LA_BF16 && fmap == LA_FMAP_ELU1 && dqk == 64 && dv == 64) return Path::FwdSplit;
    if (tc_forward_shape(dqk, dv, fmap, dtype)) return Path::FwdTc;
    return Path::FwdSimt;
}

// Sequence split of the tensor-core forward: P segments of cps chunks each,
// so that B*H*P thread blocks roughly fill the 148 SMs.
constexpr int kNumSms = 148;
constexpr int kChunk = 128;

void tc_segments(int B, int H, int N, int *P, int *cps, int *nchunks)
{
    const int BH = B * H;
    const int nc = (N + kChunk - 1) / kChunk;
    int p = kNumSms / BH;
    if (p < 1) p = 1;
    if (p > nc) p = nc;
    const int c = (nc + p - 1) / p;
    *cps = c;
    *P = (nc + c - 1) / c;
    *nchunks = nc;
}

// Chunk ranges of the split forward: T chunks of all heads in (head, chunk)
// order cut into G contiguous ranges, one per block, G <= 148 and at most
// SplitCfg64::MAX_PER_HEAD ranges per head.
void split_grid(int B, int H, int N, long long *T, int *G, int *nc)
{
    const long long BH = (long long)B * H;
    *nc = (N + kChunk - 1) / kChunk;
    *T = BH * *nc;
    long long g = *T < kNumSms ? *T : kNumSms;
    if (g > BH * SplitCfg64::MAX_PER_HEAD) g = BH * SplitCfg64::MAX_PER_HEAD;
    *G = (int)g;
}

// Workspace of the split forward: per-chunk phi(K) tiles, per-chunk
// snapshots, then two fp32 aggregates per range.
size_t split_phik_bytes(long long T) { return (size_t)T * SplitCfg64::TILE; }
size_t split_snap_bytes(long long T) { return (size_t)T * SplitCfg64::SNAP; }
size_t split_ws_bytes(long long T, int G)
{
    return split_phik_bytes(T) + split_snap_bytes(T) + (size_t)G * 2 * SplitCfg64::AGG * sizeof(float);
}

// fp32 elements per segment increment: FP x NA.
int64_t tc_increment_floats(int dqk, int dv, int fmap)
{
    const int FP = fmap == LA_FMAP_ELU1 ? dqk : 160;
    return (int64_t)FP * (dv + 16);
}

// Which tensor-core backward serves a shape: 0 none, 1 elu d = 128,
// 2 elu d = 64, 3 Taylor d' = 16 with d_v = 64 (either Taylor map).
int bwd_tc_kind(int dqk, int dv, int fmap, int dtype)
{
    if (dtype != LA_BF16) return 0;
    if (fmap == LA_FMAP_ELU1 && dqk == 128 && dv == 128) return 1;
    if (fmap == LA_FMAP_ELU1 && dqk == 64 && dv == 64) return 2;
    if (fmap != LA_FMAP_ELU1 && dqk == 16 && dv == 64) return 3;
    return 0;
}

// fp32 elements of one segment increment (S or R) of the tensor-core backward.
size_t bwd_increment_floats(int kind)
{
    switch (kind) {
    case 1: return (size_t)BwdCfg128::F * BwdCfg128::NA;
    case 2: return (size_t)BwdCfg64::F * BwdCfg64::NA;
    case 3: return (size_t)BwdCfgT16::F * BwdCfgT16::NA;
    default: return 0;
    }
}

Path select_backward(int B, int H, int N, int dqk, int dv, int fmap, int dtype)
{
    if (check_shape(B, H, N, dqk, dv, fmap, dtype) != LA_OK) return Path::Invalid;
    if (bwd_tc_kind(dqk, dv, fmap, dtype)) return Path::BwdTc;
    return Path::BwdSimt;
}

Path select_decode(int B, int H, int dqk, int dv, int fmap, int dtype)
{
    if (check_shape(B, H, 1, dqk, dv, fmap, dtype) != LA_OK) return Path::Invalid;
    if (dv == 32 || dv == 64 || dv == 128) return Path::DecodeVec;
    return Path::DecodeSimt;
}

// Kernel names and launch count of a path.
int path_kernels(Path p, const char **names)
{
    switch (p) {
    case Path::FwdSimt: names[0] = "fwd_simt_kernel"; return 1;
    case Path::FwdSplit: names[0] = "fwd_split_state_kernel"; names[1] = "fwd_split_out_kernel"; return 2;
    case Path::FwdTc: names[0] = "fwd_tc_kernel"; return 1;  // plus the segment pass, see below
    case Path::BwdSimt: names[0] = "bwd_simt_kernel"; return 1;
    case Path::BwdTc: names[0] = "bwd_dq_kernel"; names[1] = "bwd_dkdv_kernel"; return 2;
    case Path::DecodeSimt: names[0] = "decode_simt_kernel"; return 1;
    case Path::DecodeVec: names[0] = "decode_vec_kernel"; return 1;
    default: return -1;
    }
}

// Largest chunk length in {32, 16, 8, 4} whose shared-memory footprint fits.
template <typename Layout, typename MakeLayout>
bool pick_chunk(MakeLayout make, int F, int dqk, int dv, Layout *out, size_t *bytes)
{
    for (int C = 32; C >= 4; C /= 2) {
        Layout L = make(C, F, dv);
        const size_t b = L.floats(F, dqk, dv) * sizeof(float);
        if (b <= kSmemLimit) {
            *out = L;
            *bytes = b;
            return true;
        }
    }
    return false;
}

template <typename T>
la_status forward_simt(const void *q, const void *k, const void *v, void *o, const float *s_in,
                       const float *z_in, float *s_out, float *z_out, float *den_out, int B, int H, int N,
                       int dqk, int dv, int fmap, cudaStream_t stream, const int *cu = nullptr, int T_total = 0,
                       const float *logdecay = nullptr)
{
    const FmapParams fp = make_fmap(fmap, dqk);
    SimtFwdSmem L;
    size_t bytes;
    if (!pick_chunk(simt_fwd_layout, fp.F, dqk, dv, &L, &bytes)) return LA_ERR_UNSUPPORTED;
    if (set_smem<fwd_simt_kernel<T>>(bytes) != LA_OK) return LA_ERR_CUDA;
    fwd_simt_kernel<T><<<B * H, kSimtThreads, bytes, stream>>>(
        (const T *)q, (const T *)k, (const T *)v, (T *)o, s_in, z_in, s_out, z_out, den_out, N, dv, fp, L, cu, H,
        T_total, logdecay);
    return launch_status();
}

template <typename T>
la_status backward_simt(const void *q, const void *k, const void *v, const void *dout, void *dq,
                        void *dk, void *dvp, float *ws, int B, int H, int N, int dqk, int dv,
                        int fmap, cudaStream_t stream, const float *logdecay = nullptr,
                        float *dlogdecay = nullptr)
{
    // The backward reads no state, and both Taylor maps give the same
    // phi(q).phi(k), hence the same gradients: run the 273-feature map on the
    // folded features (1 + 2d' + d'(d'-1)/2 of them), 44 % less work.
    const FmapParams fp = make_fmap(fmap == LA_FMAP_TAYLOR2 ? LA_FMAP_TAYLOR2_SYM : fmap, dqk);
    SimtBwdSmem L;
    size_t bytes;
    if (!pick_chunk(simt_bwd_layout, fp.F, dqk, dv, &L, &bytes)) return LA_ERR_UNSUPPORTED;
    if (set_smem<bwd_simt_kernel<T>>(bytes) != LA_OK) return LA_ERR_CUDA;
    bwd_simt_kernel<T><<<B * H, kSimtThreads, bytes, stream>>>(
        (const T *)q, (const T *)k, (const T *)v, (const T *)dout, ws, (T *)dq, (T *)dk, (T *)dvp,
        N, dv, fp, L, logdecay, dlogdecay);
    return launch_status();
}

template <typename T>
la_status decode_simt(const void *q, const void *k, const void *v, void *y, float *s, float *z,
                      int B, int H, int dqk, int dv, int fmap, cudaStream_t stream, const float *g = nullptr)
{
    const FmapParams fp = make_fmap(fmap, dqk);
    const int R = kSimtThreads / dv;
    const int threads = R * dv;
    const size_t bytes = sizeof(float) * (2 * (size_t)fp.F + 2 * dqk + dv + (size_t)R * dv + 32);
    if (set_smem<decode_simt_kernel<T>>(bytes) != LA_OK) return LA_ERR_CUDA;
    decode_simt_kernel<T><<<B * H, threads, bytes, stream>>>((const T *)q, (const T *)k,
                                                             (const T *)v, (T *)y, s, z, dv, fp, g);
    return launch_status();
}

template <typename T>
la_status decode_vec(const void *q, const void *k, const void *v, void *y, float *s, float *z,
                     int B, int H, int dqk, int dv, int fmap, cudaStream_t stream, const float *g = nullptr)
{
    const FmapParams fp = make_fmap(fmap, dqk);
    const T *qq = (const T *)q, *kk = (const T *)k, *vv = (const T *)v;
    T *yy = (T *)y;
    // state rows per pass: 256 threads / (dv / 4) float4 groups per row
    const int passes = (fp.F + kDecodeThreads / (dv / 4) - 1) / (kDecodeThreads / (dv / 4));
    const bool short_state = passes <= 10;
    auto go = [&](auto kernel) { return launch_pdl(kernel, B * H, kDecodeThreads, 0, stream, qq, kk, vv, yy, s, z, fp, g); };
    switch (dv) {
    case 32: return short_state ? go(decode_vec_kernel<T, 32, 10, 3>) : go(decode_vec_kernel<T, 32, 18, 2>);
    case 64: return short_state ? go(decode_vec_kernel<T, 64, 10, 3>) : go(decode_vec_kernel<T, 64, 18, 2>);
    case 128: return short_state ? go(decode_vec_kernel<T, 128, 10, 3>) : go(decode_vec_kernel<T, 128, 18, 2>);
    default: return LA_ERR_UNSUPPORTED;
    }
}

// ---------------------------------------------------------- tensor maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 3D bf16 view [BH][N][inner] of a dense row-major tensor, box
// {box_inner, 128, 1}; rows past N read as zero.
bool make_map(CUtensorMap *m, const void *base, int inner, int N, int BH, int box_inner,
              CUtensorMapSwizzle sw, int box_rows = kChunk)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)N * inner * 2};
    cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The segment-state launch (P > 1) and the main launch of fwd_tc_kernel.
template <class Cfg, bool GATED>
la_status forward_tc_run(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &to,
                         const FwdParams &p, int BH, cudaStream_t stream)
{
    if (set_smem<fwd_tc_kernel<Cfg, 0, GATED>>(Cfg::SMEM_ALLOC) != LA_OK) return LA_ERR_CUDA;
    if (p.P > 1) {
        if (set_smem<fwd_tc_kernel<Cfg, 1, GATED>>(Cfg::SMEM_ALLOC) != LA_OK) return LA_ERR_CUDA;
        if (launch_pdl(fwd_tc_kernel<Cfg, 1, GATED>, BH * p.P, 288, Cfg::SMEM_ALLOC, stream, tq, tk, tv, to, p) != LA_OK)
            return LA_ERR_CUDA;
    }
    return launch_pdl(fwd_tc_kernel<Cfg, 0, GATED>, BH * p.P, 288, Cfg::SMEM_ALLOC, stream, tq, tk, tv, to, p);
}

template <class Cfg>
la_status forward_tc_launch(const void *q, const void *k, const void *v, void *o, const float *s_in,
                            const float *z_in, float *s_out, float *z_out, float *den_out, void *workspace, int B,
                            int H, int N, cudaStream_t stream, bool sym_state = false, const int *cu = nullptr,
                            int T = 0, const float *logdecay = nullptr)
{
    // Fixed length: B*H slices of N tokens, tensors [B*H, N, *].  Packed
    // sequences (cu != null): B sequences of at most N tokens, tensors [H, T, *].
    const int BH = B * H;
    const int map_rows = cu ? T : N, map_slices = cu ? H : BH;
    CUtensorMap tq, tk, tv, to;
    const CUtensorMapSwizzle qsw = Cfg::TAYLOR ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B;
    const int qbox = Cfg::TAYLOR ? 16 : 64;
    if (!make_map(&tq, q, Cfg::DQK, map_rows, map_slices, qbox, qsw) ||
        !make_map(&tk, k, Cfg::DQK, map_rows, map_slices, qbox, qsw) ||
        !make_map(&tv, v, Cfg::DV, map_rows, map_slices, 16, CU_TENSOR_MAP_SWIZZLE_32B))
        return LA_ERR_CUDA;
    // y leaves by TMA stores of 64-column SW128 boxes ([BH, N, DV], or the
    // packed [H, T, DV])
    if (!make_map(&to, o, Cfg::DV, map_rows, map_slices, 64, CU_TENSOR_MAP_SWIZZLE_128B)) return LA_ERR_CUDA;
    FwdParams p;
    p.s_in = s_in;
    p.z_in = z_in;
    p.s_out = s_out;
    p.z_out = z_out;
    p.den_out = den_out;
    p.sym_state = sym_state ? 1 : 0;
    p.ws = (float *)workspace;
    p.o = o;
    p.N = N;
    p.cu = cu;
    p.H = H;
    p.T = T;
    p.max_len = N;
    p.logdecay = logdecay;
    tc_segments(B, H, N, &p.P, &p.cps, &p.nchunks);
    const double d = (double)Cfg::DQK;
    p.inv_c1 = (float)(1.0 / pow(d, 0.25));
    p.inv_c2 = (float)(1.0 / (sqrt(2.0) * sqrt(d)));
    p.k1 = (float)(1.0 / sqrt(d));
    p.k2 = (float)(1.0 / (2.0 * d));
    if (logdecay) return forward_tc_run<Cfg, true>(tq, tk, tv, to, p, BH, stream);
    return forward_tc_run<Cfg, false>(tq, tk, tv, to, p, BH, stream);
}

// Chunk-parallel forward (elu, d_qk = d_v = 64): state launch, then output launch.
la_status forward_split64(const void *q, const void *k, const void *v, void *o, const float *s_in,
                          const float *z_in, float *s_out, float *z_out,
                          float *den_out, void *workspace, int B, int H, int N, cudaStream_t stream)
{
    const int BH = B * H;
    CUtensorMap tq, tk, tv, to;
    if (!make_map(&tq, q, 64, N, BH, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tk, k, 64, N, BH, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tv, v, 64, N, BH, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&to, o, 64, N, BH, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return LA_ERR_CUDA;
    SplitParams p;
    split_grid(B, H, N, &p.T, &p.G, &p.nc);
    p.s_in = s_in;
    p.z_in = z_in;
    p.o = (__nv_bfloat16 *)o;
    p.den_out = den_out;
    p.s_out = s_out;
    p.z_out = z_out;
    p.phik = (uint8_t *)workspace;
    p.snap = p.phik + split_phik_bytes(p.T);
    p.agg = (float *)(p.snap + split_snap_bytes(p.T));
    p.N = N;
    using Cfg = SplitCfg64;
    if (set_smem<fwd_split_state_kernel>(Cfg::S_SMEM_ALLOC) != LA_OK ||
        set_smem<fwd_split_out_kernel>(Cfg::O_SMEM_ALLOC) != LA_OK) {
#ifdef LA_DEBUG_LAUNCH
        fprintf(stderr, "libla: shared-memory attribute of the split forward refused\n");
#endif
        return LA_ERR_CUDA;
    }
    // Both launches are programmatic dependents of the kernel before them in
    // the stream: the state launch sets up on SMs the previous kernel has left
    // and waits for it to complete before touching global memory; the output
    // launch may start on SMs the state launch has left and waits for the
    // state launch before using its results.
    if (launch_pdl(fwd_split_state_kernel, p.G, Cfg::S_THREADS, Cfg::S_SMEM_ALLOC, stream, tk, tv, p) != LA_OK)
        return LA_ERR_CUDA;
    return launch_pdl(fwd_split_out_kernel, p.G, Cfg::O_THREADS, Cfg::O_SMEM_ALLOC, stream, tq, tv, to, p);
}

la_status forward_tc(const void *q, const void *k, const void *v, void *o, const float *s_in, const float *z_in,
                     float *s_out, float *z_out,
                     float *den_out, void *workspace, int B, int H, int N, int dqk, int dv, int fmap,
                     cudaStream_t stream, const int *cu = nullptr, int T = 0, const float *logdecay = nullptr)
{
    if (fmap != LA_FMAP_ELU1)
        return forward_tc_launch<FwdCfg<16, 64, true>>(q, k, v, o, s_in, z_in, s_out, z_out, den_out, workspace, B, H, N,
                                                       stream, fmap == LA_FMAP_TAYLOR2_SYM, cu, T, logdecay);
    if (dqk == 64)
        return forward_tc_launch<FwdCfg<64, 64, false>>(q, k, v, o, s_in, z_in, s_out, z_out, den_out, workspace, B, H,
                                                        N, stream, false, cu, T, logdecay);
    return forward_tc_launch<FwdCfg<128, 128, false>>(q, k, v, o, s_in, z_in, s_out, z_out, den_out, workspace, B, H,
                                                      N, stream, false, cu, T, logdecay);
}

// Workspace of the tensor-core backward (floats): den_i, dden_i per token;
// gated, c_i per token; when P > 1, the S and R increments per segment and,
// gated, each segment's summed gate.
template <class Cfg, bool GATED>
la_status backward_tc(const void *q, const void *k, const void *v, const void *dout, void *dq, void *dk,
                      void *dvp, void *workspace, int B, int H, int N, cudaStream_t stream,
                      const float *log_decay = nullptr, float *dlog_decay = nullptr)
{
    const int BH = B * H;
    CUtensorMap tq, tk, tv, tdo, tdq, tdk, tdv;
    const int qbox = Cfg::TAYLOR ? 16 : 64;
    const CUtensorMapSwizzle qsw = Cfg::TAYLOR ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B;
    // dq and dk leave through maps of Q's and K's geometry (stores of the tiles
    // their inputs were loaded into)
    if (!make_map(&tq, q, Cfg::D, N, BH, qbox, qsw) || !make_map(&tk, k, Cfg::D, N, BH, qbox, qsw) ||
        !make_map(&tv, v, Cfg::DV, N, BH, 16, CU_TENSOR_MAP_SWIZZLE_32B) ||
        !make_map(&tdo, dout, Cfg::DV, N, BH, 16, CU_TENSOR_MAP_SWIZZLE_32B) ||
        !make_map(&tdq, dq, Cfg::D, N, BH, qbox, qsw) || !make_map(&tdk, dk, Cfg::D, N, BH, qbox, qsw) ||
        !make_map(&tdv, dvp, Cfg::DV, N, BH, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return LA_ERR_CUDA;
    BwdParams p;
    tc_segments(B, H, N, &p.P, &p.cps, &p.nchunks);
    p.N = N;
    p.dd = (float *)workspace;
    p.cvec = p.dd + (size_t)BH * N * 2;
    float *ws_s = p.cvec + (GATED ? (size_t)BH * N : 0);
    float *ws_r = ws_s + (size_t)BH * p.P * Cfg::F * Cfg::NA;
    p.ws_s = ws_s;
    p.ws_r = ws_r;
    p.ws_log = ws_r + (size_t)BH * p.P * Cfg::F * Cfg::NA;
    p.logdecay = log_decay;
    p.dg = dlog_decay;
    p.dq = dq;
    p.dk = dk;
    p.dv = dvp;
    const double d = (double)Cfg::D;
    p.inv_c1 = (float)(1.0 / pow(d, 0.25));
    p.inv_c2 = (float)(1.0 / (sqrt(2.0) * sqrt(d)));
    p.inv_c3 = (float)(1.0 / sqrt(d));
    p.k2 = (float)(1.0 / (2.0 * d));
    // the S and R increment passes: elu on the three-stage kernels, Taylor on
    // the two-stage ones (its phi tile is built from the raw tile in place)
    auto state_pass = [&](bool s_pass) -> la_status {
        if constexpr (Cfg::TAYLOR) {
            if (s_pass) {
                if (set_smem<bwd_sstate_kernel<Cfg, GATED>>(Cfg::SMEM_ALLOC) != LA_OK) return LA_ERR_CUDA;
                bwd_sstate_kernel<Cfg, GATED><<<BH * p.P, 128, Cfg::SMEM_ALLOC, stream>>>(tk, tv, p);
            } else {
                if (set_smem<bwd_rstate_kernel<Cfg, GATED>>(Cfg::SMEM_ALLOC) != LA_OK) return LA_ERR_CUDA;
                bwd_rstate_kernel<Cfg, GATED><<<BH * p.P, 128, Cfg::SMEM_ALLOC, stream>>>(tq, tdo, p);
            }
        } else {
            if (s_pass) {
                if (set_smem<bwd_sstate3_kernel<Cfg, GATED>>(Cfg::SP_SMEM) != LA_OK) return LA_ERR_CUDA;
                bwd_sstate3_kernel<Cfg, GATED><<<BH * p.P, 256, Cfg::SP_SMEM, stream>>>(tk, tv, p);
            } else {
                if (set_smem<bwd_rstate3_kernel<Cfg, GATED>>(Cfg::SP_SMEM) != LA_OK) return LA_ERR_CUDA;
                bwd_rstate3_kernel<Cfg, GATED><<<BH * p.P, 256, Cfg::SP_SMEM, stream>>>(tq, tdo, p);
            }
        }
        return launch_status();
    };
    if (p.P > 1 && state_pass(true) != LA_OK) return LA_ERR_CUDA;
    if (set_smem<bwd_dq_kernel<Cfg, GATED>>(Cfg::SMEM_ALLOC) != LA_OK ||
        set_smem<bwd_dkdv_kernel<Cfg, GATED>>(Cfg::SMEM_ALLOC) != LA_OK)
        return LA_ERR_CUDA;
    bwd_dq_kernel<Cfg, GATED><<<BH * p.P, 256, Cfg::SMEM_ALLOC, stream>>>(tq, tk, tv, tdo, tdq, p);
    if (launch_status() != LA_OK) return LA_ERR_CUDA;
    if (p.P > 1 && state_pass(false) != LA_OK) return LA_ERR_CUDA;
    bwd_dkdv_kernel<Cfg, GATED><<<BH * p.P, 256, Cfg::SMEM_ALLOC, stream>>>(tq, tk, tv, tdo, tdk, tdv, p);
    if (!GATED) return launch_status();
    if (launch_status() != LA_OK) return LA_ERR_CUDA;
    bwd_dg_kernel<<<BH, 1024, 0, stream>>>(p.cvec, p.dg, N);
    return launch_status();
}

// One warp; lane 0 waits on an mbarrier that expects one arrival nobody
// makes, through the kernels' bounded wait with a caller-chosen limit.
__global__ void selftest_wait_kernel(uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::mbar_init_fence();
        sm100::mbar_wait(&bar, 0, limit_ns);
    }
    __syncwarp();
}

}  // namespace

// ------------------------------------------------ sliding-window attention

static la_status check_swa(int B, int H, int N, int dqk, int dv, int window, int dtype)
{
    if (B < 1 || H < 1 || N < 1 || dqk < 1 || dv < 1 || window < 1) return LA_ERR_INVALID_ARG;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if ((int64_t)B * H * N * (dqk > dv ? dqk : dv) >= (int64_t)1 << 31) return LA_ERR_INVALID_ARG;
    if (dqk > 128 || dv > 128 || window > kSwaMaxWindow) return LA_ERR_UNSUPPORTED;
    return LA_OK;
}

static bool swa_tc_shape(int dqk, int dv, int window, int dtype)
{
    return dtype == LA_BF16 && dqk == 64 && dv == 64 && window % 16 == 0 && window >= 16 && window <= 128;
}

template <int W>
static la_status swa_tc_launch(const void *q, const void *k, const void *v, void *o, float *lse, int BH, int N,
                               cudaStream_t stream)
{
    using Cfg = SwaCfg<W>;
    CUtensorMap tq, tk, tv, to;
    if (!make_map(&tq, q, 64, N, BH, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tk, k, 64, N, BH, 64, CU_TENSOR_MAP_SWIZZLE_128B, Cfg::KW) ||
        !make_map(&tv, v, 64, N, BH, 64, CU_TENSOR_MAP_SWIZZLE_128B, Cfg::KW) ||
        !make_map(&to, o, 64, N, BH, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return LA_ERR_CUDA;
    SwaParams p;
    p.o = (__nv_bfloat16 *)o;
    p.lse = lse;
    p.N = N;
    p.BH = BH;
    p.tiles_per_bh = (N + Cfg::C - 1) / Cfg::C;
    p.scale = (float)(1.0 / sqrt(64.0));
    p.scale_log2 = (float)(1.4426950408889634 / sqrt(64.0));
    const long long ntiles = (long long)BH * p.tiles_per_bh;
    const int per_sm = Cfg::TMEM_COLS == 256 ? 2 : 1;   // TMEM: 512 columns per SM
    const int grid = (int)(ntiles < (long long)per_sm * kNumSms ? ntiles : per_sm * kNumSms);
    if (set_smem<swa_fwd_tc_kernel<Cfg>>(Cfg::SMEM_ALLOC) != LA_OK) return LA_ERR_CUDA;
    return launch_pdl(swa_fwd_tc_kernel<Cfg>, grid, Cfg::THREADS, Cfg::SMEM_ALLOC, stream, tq, tk, tv, to, p);
}

template <typename T>
static la_status swa_simt_launch(const void *q, const void *k, const void *v, void *o, float *lse, int BH, int N,
                                 int dqk, int dv, int window, cudaStream_t stream)
{
    const int rblocks = (N + kSwaSimtWarps - 1) / kSwaSimtWarps;
    const long long blocks = (long long)BH * rblocks;
    if (blocks >= ((long long)1 << 31)) return LA_ERR_UNSUPPORTED;
    const size_t bytes = (size_t)kSwaSimtWarps * (window + dqk) * sizeof(float);
    if (set_smem<swa_fwd_simt_kernel<T>>(bytes) != LA_OK) return LA_ERR_CUDA;
    swa_fwd_simt_kernel<T><<<(unsigned)blocks, 32 * kSwaSimtWarps, bytes, stream>>>(
        (const T *)q, (const T *)k, (const T *)v, (T *)o, lse, N, dqk, dv, window, (float)(1.0 / sqrt((double)dqk)));
    return launch_status();
}

extern "C" {

int la_version(void) { return 100; }

const char *la_status_string(int status)
{
    switch (status) {
    case LA_OK: return "LA_OK";
    case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG";
    case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED";
    case LA_ERR_CUDA: return "LA_ERR_CUDA";
    case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT";
    case LA_ERR_DEVICE_CHECK: return "LA_ERR_DEVICE_CHECK";
    case LA_ERR_SCRATCH_LIMIT: return "LA_ERR_SCRATCH_LIMIT";
    default: return "LA_ERR_UNKNOWN";
    }
}

int64_t la_feature_dim(int fmap, int dqk)
{
    if (dqk < 1) return -1;
    if (fmap == LA_FMAP_ELU1) return dqk;
    if (fmap == LA_FMAP_TAYLOR2) return 1 + (int64_t)dqk + (int64_t)dqk * dqk;
    if (fmap == LA_FMAP_TAYLOR2_SYM) return 1 + 2 * (int64_t)dqk + (int64_t)dqk * (dqk - 1) / 2;
    return -1;
}

size_t la_forward_workspace_bytes(int B, int H, int N, int dqk, int dv, int fmap, int dtype)
{
    const Path path = select_forward(B, H, N, dqk, dv, fmap, dtype);
    if (path == Path::FwdSplit) {
        long long T;
        int G, nc;
        split_grid(B, H, N, &T, &G, &nc);
        return split_ws_bytes(T, G);
    }
    if (path != Path::FwdTc) return 0;
    int P, cps, nc;
    tc_segments(B, H, N, &P, &cps, &nc);
    if (P <= 1) return 0;
    return (size_t)B * H * P * tc_increment_floats(dqk, dv, fmap) * sizeof(float);
}

size_t la_backward_workspace_bytes(int B, int H, int N, int dqk, int dv, int fmap, int dtype)
{
    const Path path = select_backward(B, H, N, dqk, dv, fmap, dtype);
    if (path == Path::Invalid) return 0;
    size_t bytes = (size_t)B * H * N * 2 * sizeof(float);  // den_i, dden_i
    if (path == Path::BwdTc) {
        int P, cps, nc;
        tc_segments(B, H, N, &P, &cps, &nc);
        if (P > 1) bytes += 2 * (size_t)B * H * P * bwd_increment_floats(bwd_tc_kind(dqk, dv, fmap, dtype)) *
                                sizeof(float);   // S, R increments
    }
    return bytes;
}

static la_status forward_impl(const void *q, const void *k, const void *v, void *o, const float *s_in,
                              const float *z_in, float *s_out, float *z_out, float *den_out, void *workspace,
                              size_t workspace_bytes, int B, int H, int N, int dqk, int dv, int fmap, int dtype,
                              void *stream)
{
    const la_status sh = check_shape(B, H, N, dqk, dv, fmap, dtype);
    if (sh != LA_OK) return sh;
    if (!q || !k || !v || !o) return LA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(s_out, 16) || !aligned(z_out, 4) || !aligned(den_out, 4))
        return LA_ERR_INVALID_ARG;
    if (check_on_current_device(q) != LA_OK) return LA_ERR_INVALID_ARG;
    if (workspace_bytes < la_forward_workspace_bytes(B, H, N, dqk, dv, fmap, dtype))
        return LA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const Path path = select_forward(B, H, N, dqk, dv, fmap, dtype);
    if (path == Path::FwdSplit) {
        if (!workspace || !aligned(workspace, 16)) return LA_ERR_INVALID_ARG;
        return forward_split64(q, k, v, o, s_in, z_in, s_out, z_out, den_out, workspace, B, H, N, s);
    }
    if (path == Path::FwdTc) {
        if (workspace_bytes && !aligned(workspace, 16)) return LA_ERR_INVALID_ARG;
        if (la_forward_workspace_bytes(B, H, N, dqk, dv, fmap, dtype) && !workspace) return LA_ERR_INVALID_ARG;
        return forward_tc(q, k, v, o, s_in, z_in, s_out, z_out, den_out, workspace, B, H, N, dqk, dv, fmap, s);
    }
    if (dtype == LA_F32)
        return forward_simt<float>(q, k, v, o, s_in, z_in, s_out, z_out, den_out, B, H, N, dqk, dv, fmap, s);
    return forward_simt<__nv_bfloat16>(q, k, v, o, s_in, z_in, s_out, z_out, den_out, B, H, N, dqk, dv, fmap, s);
}

la_status la_forward(const void *q, const void *k, const void *v, void *o, float *s_out,
                     float *z_out, float *den_out, void *workspace, size_t workspace_bytes, int B,
                     int H, int N, int dqk, int dv, int fmap, int dtype, void *stream)
{
    return forward_impl(q, k, v, o, nullptr, nullptr, s_out, z_out, den_out, workspace, workspace_bytes, B, H, N,
                        dqk, dv, fmap, dtype, stream);
}

// Byte ranges [a, a + na) and [b, b + nb) overlap (null never overlaps).
static bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    if (!a || !b) return false;
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return x < y + nb && y < x + na;
}

la_status la_forward_from_state(const void *q, const void *k, const void *v, void *o, const float *s_in,
                                const float *z_in, float *s_out, float *z_out, float *den_out, void *workspace,
                                size_t workspace_bytes, int B, int H, int N, int dqk, int dv, int fmap,
                                int dtype, void *stream)
{
    const la_status sh = check_shape(B, H, N, dqk, dv, fmap, dtype);
    if (sh != LA_OK) return sh;
    if (!s_in || !z_in || !aligned(s_in, 16) || !aligned(z_in, 4)) return LA_ERR_INVALID_ARG;
    const size_t F = (size_t)la_feature_dim(fmap, dqk);
    const size_t sb = (size_t)B * H * F * dv * sizeof(float), zb = (size_t)B * H * F * sizeof(float);
    if (overlaps(s_in, sb, s_out, sb) || overlaps(s_in, sb, z_out, zb) || overlaps(z_in, zb, s_out, sb) ||
        overlaps(z_in, zb, z_out, zb))
        return LA_ERR_INVALID_ARG;
    return forward_impl(q, k, v, o, s_in, z_in, s_out, z_out, den_out, workspace, workspace_bytes, B, H, N, dqk,
                        dv, fmap, dtype, stream);
}

size_t la_forward_varlen_workspace_bytes(int nseq, int H, int max_seqlen, int dqk, int dv, int fmap, int dtype)
{
    if (check_shape(nseq, H, max_seqlen, dqk, dv, fmap, dtype) != LA_OK) return 0;
    if (!tc_forward_shape(dqk, dv, fmap, dtype)) return 0;
    int P, cps, nc;
    tc_segments(nseq, H, max_seqlen, &P, &cps, &nc);
    if (P <= 1) return 0;
    return (size_t)nseq * H * P * tc_increment_floats(dqk, dv, fmap) * sizeof(float);
}

la_status la_forward_varlen(const void *q, const void *k, const void *v, void *o, const int32_t *cu_seqlens,
                            int nseq, int max_seqlen, int T, const float *s_in, const float *z_in, float *s_out,
                            float *z_out, float *den_out, void *workspace, size_t workspace_bytes, int H, int dqk,
                            int dv, int fmap, int dtype, void *stream)
{
    if (T < 1) return LA_ERR_INVALID_ARG;
    if (max_seqlen > T) max_seqlen = T;   // no sequence is longer than the batch
    la_status sh = check_shape(nseq, H, max_seqlen, dqk, dv, fmap, dtype);
    if (sh != LA_OK) return sh;
    sh = check_shape(1, H, T, dqk, dv, fmap, dtype);   // element counts of the packed tensors
    if (sh != LA_OK) return sh;
    if (!q || !k || !v || !o || !cu_seqlens || !aligned(cu_seqlens, 4)) return LA_ERR_INVALID_ARG;
    if (check_on_current_device(q) != LA_OK) return LA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(s_out, 16) ||
        !aligned(z_out, 4) || !aligned(den_out, 4))
        return LA_ERR_INVALID_ARG;
    if ((s_in == nullptr) != (z_in == nullptr)) return LA_ERR_INVALID_ARG;
    const size_t F = (size_t)la_feature_dim(fmap, dqk);
    if (s_in) {
        if (!aligned(s_in, 16) || !aligned(z_in, 4)) return LA_ERR_INVALID_ARG;
        const size_t sb = (size_t)nseq * H * F * dv * sizeof(float), zb = (size_t)nseq * H * F * sizeof(float);
        if (overlaps(s_in, sb, s_out, sb) || overlaps(s_in, sb, z_out, zb) || overlaps(z_in, zb, s_out, sb) ||
            overlaps(z_in, zb, z_out, zb))
            return LA_ERR_INVALID_ARG;
    }
    const size_t need = la_forward_varlen_workspace_bytes(nseq, H, max_seqlen, dqk, dv, fmap, dtype);
    if (workspace_bytes < need || (need && (!workspace || !aligned(workspace, 16)))) return LA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (tc_forward_shape(dqk, dv, fmap, dtype))
        return forward_tc(q, k, v, o, s_in, z_in, s_out, z_out, den_out, workspace, nseq, H, max_seqlen, dqk, dv,
                          fmap, st, cu_seqlens, T);
    if (dtype == LA_F32)
        return forward_simt<float>(q, k, v, o, s_in, z_in, s_out, z_out, den_out, nseq, H, max_seqlen, dqk, dv,
                                   fmap, st, cu_seqlens, T);
    return forward_simt<__nv_bfloat16>(q, k, v, o, s_in, z_in, s_out, z_out, den_out, nseq, H, max_seqlen, dqk, dv,
                                       fmap, st, cu_seqlens, T);
}

// Allocation-free forward: la_forward with its workspace taken from a
// scratch array compiled into the library.  Callers without access to a
// device allocator (a plugin inside a host program that owns all device
// memory, a fixed-footprint service) use it instead of allocating the
// workspace themselves.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch for the current device, looked up once
// per device.  In host code the symbol itself is only a host-side stand-in,
// so kernels must be given this address, never the symbol.
static la_status noalloc_scratch(void **out)
{
    static void *addr[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LA_ERR_CUDA;
        addr[dev] = p;
    }
    *out = addr[dev];
    return LA_OK;
}

la_status la_forward_noalloc(const void *q, const void *k, const void *v, void *o, float *s_out,
                             float *z_out, float *den_out, int B, int H, int N, int dqk, int dv,
                             int fmap, int dtype, void *stream)
{
    const la_status sh = check_shape(B, H, N, dqk, dv, fmap, dtype);
    if (sh != LA_OK) return sh;
    const size_t need = la_forward_workspace_bytes(B, H, N, dqk, dv, fmap, dtype);
    if (need > LA_NOALLOC_SCRATCH_BYTES) return LA_ERR_SCRATCH_LIMIT;
    if (need == 0)
        return la_forward(q, k, v, o, s_out, z_out, den_out, nullptr, 0, B, H, N, dqk, dv, fmap, dtype, stream);
    void *scratch = nullptr;
    const la_status st = noalloc_scratch(&scratch);
    if (st != LA_OK) return st;
    return la_forward(q, k, v, o, s_out, z_out, den_out, scratch, LA_NOALLOC_SCRATCH_BYTES, B, H, N, dqk,
                      dv, fmap, dtype, stream);
}

la_status la_backward(const void *q, const void *k, const void *v, const void *dout, void *dq,
                      void *dk, void *dvp, void *workspace, size_t workspace_bytes, int B, int H,
                      int N, int dqk, int dv, int fmap, int dtype, void *stream)
{
    const la_status sh = check_shape(B, H, N, dqk, dv, fmap, dtype);
    if (sh != LA_OK) return sh;
    if (!q || !k || !v || !dout || !dq || !dk || !dvp || !workspace) return LA_ERR_INVALID_ARG;
    if (check_on_current_device(q) != LA_OK) return LA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dout, 16) ||
        !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dvp, 16) || !aligned(workspace, 16))
        return LA_ERR_INVALID_ARG;
    if (workspace_bytes < la_backward_workspace_bytes(B, H, N, dqk, dv, fmap, dtype))
        return LA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    float *ws = (float *)workspace;
    switch (select_backward(B, H, N, dqk, dv, fmap, dtype) == Path::BwdTc ? bwd_tc_kind(dqk, dv, fmap, dtype) : 0) {
    case 1: return backward_tc<BwdCfg128, false>(q, k, v, dout, dq, dk, dvp, workspace, B, H, N, s);
    case 2: return backward_tc<BwdCfg64, false>(q, k, v, dout, dq, dk, dvp, workspace, B, H, N, s);
    case 3: return backward_tc<BwdCfgT16, false>(q, k, v, dout, dq, dk, dvp, workspace, B, H, N, s);
    default: break;
    }
    if (dtype == LA_F32)
        return backward_simt<float>(q, k, v, dout, dq, dk, dvp, ws, B, H, N, dqk, dv, fmap, s);
    return backward_simt<__nv_bfloat16>(q, k, v, dout, dq, dk, dvp, ws, B, H, N, dqk, dv, fmap, s);
}

static la_status decode_impl(const void *q, const void *k, const void *v, const float *g, void *y, float *s,
                             float *z, int B, int H, int dqk, int dv, int fmap, int dtype, void *stream)
{
    const la_status sh = check_shape(B, H, 1, dqk, dv, fmap, dtype);
    if (sh != LA_OK) return sh;
    if (!q || !k || !v || !y || !s || !z) return LA_ERR_INVALID_ARG;
    if (check_on_current_device(s) != LA_OK) return LA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(y, 16) ||
        !aligned(s, 16) || !aligned(z, 4) || !aligned(g, 4))
        return LA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (select_decode(B, H, dqk, dv, fmap, dtype) == Path::DecodeVec) {
        if (dtype == LA_F32) return decode_vec<float>(q, k, v, y, s, z, B, H, dqk, dv, fmap, st, g);
        return decode_vec<__nv_bfloat16>(q, k, v, y, s, z, B, H, dqk, dv, fmap, st, g);
    }
    if (dtype == LA_F32) return decode_simt<float>(q, k, v, y, s, z, B, H, dqk, dv, fmap, st, g);
    return decode_simt<__nv_bfloat16>(q, k, v, y, s, z, B, H, dqk, dv, fmap, st, g);
}

la_status la_decode_step(const void *q, const void *k, const void *v, void *y, float *s,
                         float *z, int B, int H, int dqk, int dv, int fmap, int dtype,
                         void *stream)
{
    return decode_impl(q, k, v, nullptr, y, s, z, B, H, dqk, dv, fmap, dtype, stream);
}

la_status la_decode_step_decay(const void *q, const void *k, const void *v, const float *log_decay, void *y,
                               float *s, float *z, int B, int H, int dqk, int dv, int fmap, int dtype,
                               void *stream)
{
    if (!log_decay) return LA_ERR_INVALID_ARG;
    return decode_impl(q, k, v, log_decay, y, s, z, B, H, dqk, dv, fmap, dtype, stream);
}

size_t la_forward_decay_workspace_bytes(int B, int H, int N, int dqk, int dv, int fmap, int dtype)
{
    if (check_shape(B, H, N, dqk, dv, fmap, dtype) != LA_OK || !tc_forward_shape(dqk, dv, fmap, dtype)) return 0;
    int P, cps, nc;
    tc_segments(B, H, N, &P, &cps, &nc);
    if (P <= 1) return 0;
    // segment increments, then each segment's sum of log gates
    return (size_t)B * H * P * (tc_increment_floats(dqk, dv, fmap) + 1) * sizeof(float);
}

size_t la_backward_decay_workspace_bytes(int B, int H, int N, int dqk, int dv, int fmap, int dtype)
{
    if (check_shape(B, H, N, dqk, dv, fmap, dtype) != LA_OK) return 0;
    const size_t BHN = (size_t)B * H * N;
    const int kind = bwd_tc_kind(dqk, dv, fmap, dtype);
    if (!kind) return BHN * 2 * sizeof(float);   // den_i, dden_i per token
    // tensor cores: den_i, dden_i and c_i per token; per segment (P > 1) the S
    // and R increments and the segment's summed gate
    int P, cps, nc;
    tc_segments(B, H, N, &P, &cps, &nc);
    size_t floats = BHN * 3;
    if (P > 1) floats += (size_t)B * H * P * (2 * bwd_increment_floats(kind) + 1);
    return floats * sizeof(float);
}

la_status la_backward_decay(const void *q, const void *k, const void *v, const float *log_decay,
                            const void *dout, void *dq, void *dk, void *dvp, float *dlog_decay, void *workspace,
                            size_t workspace_bytes, int B, int H, int N, int dqk, int dv, int fmap, int dtype,
                            void *stream)
{
    const la_status sh = check_shape(B, H, N, dqk, dv, fmap, dtype);
    if (sh != LA_OK) return sh;
    if (!q || !k || !v || !log_decay || !dout || !dq || !dk || !dvp || !dlog_decay || !workspace)
        return LA_ERR_INVALID_ARG;
    if (check_on_current_device(q) != LA_OK) return LA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dout, 16) || !aligned(dq, 16) ||
        !aligned(dk, 16) || !aligned(dvp, 16) || !aligned(log_decay, 4) || !aligned(dlog_decay, 4) ||
        !aligned(workspace, 4))
        return LA_ERR_INVALID_ARG;
    if (workspace_bytes < la_backward_decay_workspace_bytes(B, H, N, dqk, dv, fmap, dtype)) return LA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    float *ws = (float *)workspace;
    switch (bwd_tc_kind(dqk, dv, fmap, dtype)) {
    case 1: return backward_tc<BwdCfg128, true>(q, k, v, dout, dq, dk, dvp, workspace, B, H, N, st, log_decay, dlog_decay);
    case 2: return backward_tc<BwdCfg64, true>(q, k, v, dout, dq, dk, dvp, workspace, B, H, N, st, log_decay, dlog_decay);
    case 3: return backward_tc<BwdCfgT16, true>(q, k, v, dout, dq, dk, dvp, workspace, B, H, N, st, log_decay, dlog_decay);
    default: break;
    }
    if (dtype == LA_F32)
        return backward_simt<float>(q, k, v, dout, dq, dk, dvp, ws, B, H, N, dqk, dv, fmap, st, log_decay, dlog_decay);
    return backward_simt<__nv_bfloat16>(q, k, v, dout, dq, dk, dvp, ws, B, H, N, dqk, dv, fmap, st, log_decay,
                                        dlog_decay);
}

la_status la_forward_decay(const void *q, const void *k, const void *v, const float *log_decay, void *o,
                           const float *s_in, const float *z_in, float *s_out, float *z_out, float *den_out,
                           void *workspace, size_t workspace_bytes, int B, int H, int N, int dqk, int dv,
                           int fmap, int dtype, void *stream)
{
    const la_status sh = check_shape(B, H, N, dqk, dv, fmap, dtype);
    if (sh != LA_OK) return sh;
    if (!q || !k || !v || !o || !log_decay) return LA_ERR_INVALID_ARG;
    if (check_on_current_device(q) != LA_OK) return LA_ERR_INVALID_ARG;
    const size_t need = la_forward_decay_workspace_bytes(B, H, N, dqk, dv, fmap, dtype);
    if (workspace_bytes < need || (need && (!workspace || !aligned(workspace, 16)))) return LA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(log_decay, 4) ||
        !aligned(s_out, 16) || !aligned(z_out, 4) || !aligned(den_out, 4))
        return LA_ERR_INVALID_ARG;
    if ((s_in == nullptr) != (z_in == nullptr)) return LA_ERR_INVALID_ARG;
    if (s_in) {
        if (!aligned(s_in, 16) || !aligned(z_in, 4)) return LA_ERR_INVALID_ARG;
        const size_t F = (size_t)la_feature_dim(fmap, dqk);
        const size_t sb = (size_t)B * H * F * dv * sizeof(float), zb = (size_t)B * H * F * sizeof(float);
        if (overlaps(s_in, sb, s_out, sb) || overlaps(s_in, sb, z_out, zb) || overlaps(z_in, zb, s_out, sb) ||
            overlaps(z_in, zb, z_out, zb))
            return LA_ERR_INVALID_ARG;
    }
    cudaStream_t st = (cudaStream_t)stream;
    if (tc_forward_shape(dqk, dv, fmap, dtype))
        return forward_tc(q, k, v, o, s_in, z_in, s_out, z_out, den_out, workspace, B, H, N, dqk, dv, fmap, st,
                          nullptr, 0, log_decay);
    if (dtype == LA_F32)
        return forward_simt<float>(q, k, v, o, s_in, z_in, s_out, z_out, den_out, B, H, N, dqk, dv, fmap, st,
                                   nullptr, 0, log_decay);
    return forward_simt<__nv_bfloat16>(q, k, v, o, s_in, z_in, s_out, z_out, den_out, B, H, N, dqk, dv, fmap, st,
                                       nullptr, 0, log_decay);
}

la_status la_swa_forward(const void *q, const void *k, const void *v, void *o, float *lse_out, int B, int H, int N,
                         int dqk, int dv, int window, int dtype, void *stream)
{
    const la_status sh = check_swa(B, H, N, dqk, dv, window, dtype);
    if (sh != LA_OK) return sh;
    if (!q || !k || !v || !o) return LA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse_out, 4))
        return LA_ERR_INVALID_ARG;
    if (check_on_current_device(q) != LA_OK) return LA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const int BH = B * H;
    if (swa_tc_shape(dqk, dv, window, dtype)) {
        switch (window) {
        case 16: return swa_tc_launch<16>(q, k, v, o, lse_out, BH, N, st);
        case 32: return swa_tc_launch<32>(q, k, v, o, lse_out, BH, N, st);
        case 48: return swa_tc_launch<48>(q, k, v, o, lse_out, BH, N, st);
        case 64: return swa_tc_launch<64>(q, k, v, o, lse_out, BH, N, st);
        case 80: return swa_tc_launch<80>(q, k, v, o, lse_out, BH, N, st);
        case 96: return swa_tc_launch<96>(q, k, v, o, lse_out, BH, N, st);
        case 112: return swa_tc_launch<112>(q, k, v, o, lse_out, BH, N, st);
        default: return swa_tc_launch<128>(q, k, v, o, lse_out, BH, N, st);
        }
    }
    if (dtype == LA_F32) return swa_simt_launch<float>(q, k, v, o, lse_out, BH, N, dqk, dv, window, st);
    return swa_simt_launch<__nv_bfloat16>(q, k, v, o, lse_out, BH, N, dqk, dv, window, st);
}

int la_swa_kernel_plan(int decode, int B, int H, int N, int dqk, int dv, int window, int dtype, char *buf,
                       size_t buflen)
{
    if (check_swa(B, H, decode ? 1 : N, dqk, dv, window, dtype) != LA_OK) return -1;
    const char *nm = decode ? (dqk == 64 && dv == 64 && window <= 64 ? "swa_decode64_kernel" : "swa_decode_kernel")
                            : (swa_tc_shape(dqk, dv, window, dtype) ? "swa_fwd_tc_kernel" : "swa_fwd_simt_kernel");
    if (buf && buflen) {
        strncpy(buf, nm, buflen - 1);
        buf[buflen - 1] = 0;
    }
    return 1;
}

la_status la_swa_cache_fill(const void *k, const void *v, void *k_cache, void *v_cache, int B, int H, int N,
                            int dqk, int dv, int window, int dtype, void *stream)
{
    const la_status sh = check_swa(B, H, N, dqk, dv, window, dtype);
    if (sh != LA_OK) return sh;
    if (!k || !v || !k_cache || !v_cache) return LA_ERR_INVALID_ARG;
    if (check_on_current_device(k_cache) != LA_OK) return LA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (dtype == LA_F32)
        swa_cache_fill_kernel<float><<<B * H, 256, 0, st>>>((const float *)k, (const float *)v, (float *)k_cache,
                                                            (float *)v_cache, N, dqk, dv, window);
    else
        swa_cache_fill_kernel<__nv_bfloat16><<<B * H, 256, 0, st>>>(
            (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, (__nv_bfloat16 *)k_cache, (__nv_bfloat16 *)v_cache,
            N, dqk, dv, window);
    return launch_status();
}

la_status la_swa_decode_step(const void *q, const void *k, const void *v, void *y, void *k_cache, void *v_cache,
                             const int32_t *pos, int B, int H, int dqk, int dv, int window, int dtype, void *stream)
{
    const la_status sh = check_swa(B, H, 1, dqk, dv, window, dtype);
    if (sh != LA_OK) return sh;
    if (!q || !k || !v || !y || !k_cache || !v_cache || !pos || !aligned(pos, 4)) return LA_ERR_INVALID_ARG;
    if (check_on_current_device(k_cache) != LA_OK) return LA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t bytes = sizeof(float) * ((size_t)window + dqk + 8);
    const float scale = (float)(1.0 / sqrt((double)dqk));
    const bool vec = dqk == 64 && dv == 64 && window <= 64 && aligned(q, 16) && aligned(k, 16) && aligned(v, 16) &&
                     aligned(k_cache, 16) && aligned(v_cache, 16);
    if (vec) {
        if (dtype == LA_F32)
            return launch_pdl(swa_decode64_kernel<float>, B * H, 128, 0, st, (const float *)q, (const float *)k,
                              (const float *)v, (float *)y, (float *)k_cache, (float *)v_cache, pos, H, window, scale);
        return launch_pdl(swa_decode64_kernel<__nv_bfloat16>, B * H, 128, 0, st, (const __nv_bfloat16 *)q,
                          (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, (__nv_bfloat16 *)y,
                          (__nv_bfloat16 *)k_cache, (__nv_bfloat16 *)v_cache, pos, H, window, scale);
    }
    if (dtype == LA_F32) {
        if (set_smem<swa_decode_kernel<float>>(bytes) != LA_OK) return LA_ERR_CUDA;
        swa_decode_kernel<float><<<B * H, kSwaDecodeThreads, bytes, st>>>(
            (const float *)q, (const float *)k, (const float *)v, (float *)y, (float *)k_cache, (float *)v_cache, pos,
            H, dqk, dv, window, scale);
    } else {
        if (set_smem<swa_decode_kernel<__nv_bfloat16>>(bytes) != LA_OK) return LA_ERR_CUDA;
        swa_decode_kernel<__nv_bfloat16><<<B * H, kSwaDecodeThreads, bytes, st>>>(
            (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, (__nv_bfloat16 *)y,
            (__nv_bfloat16 *)k_cache, (__nv_bfloat16 *)v_cache, pos, H, dqk, dv, window, scale);
    }
    return launch_status();
}

la_status la_feature_map(const void *x, void *phi, int64_t rows, int dqk, int fmap, int dtype,
                         void *stream)
{
    if (!valid_enums(fmap, dtype) || rows < 1 || dqk < 1) return LA_ERR_INVALID_ARG;
    if (!x || !phi) return LA_ERR_INVALID_ARG;
    if (!supported_dims(fmap, dqk, 1)) return LA_ERR_UNSUPPORTED;
    if (check_on_current_device(x) != LA_OK) return LA_ERR_INVALID_ARG;
    const FmapParams fp = make_fmap(fmap, dqk);
    if (rows * fp.F >= ((int64_t)1 << 40)) return LA_ERR_INVALID_ARG;
    const int64_t total = rows * fp.F;
    const int threads = 256;
    const int64_t want = (total + threads - 1) / threads;
    const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
    cudaStream_t s = (cudaStream_t)stream;
    if (dtype == LA_F32)
        feature_map_kernel<float><<<blocks, threads, 0, s>>>((const float *)x, (float *)phi, rows, fp);
    else
        feature_map_kernel<__nv_bfloat16><<<blocks, threads, 0, s>>>(
            (const __nv_bfloat16 *)x, (__nv_bfloat16 *)phi, rows, fp);
    return launch_status();
}

int la_kernel_plan(int op, int B, int H, int N, int dqk, int dv, int fmap, int dtype, char *buf,
                   size_t buflen)
{
    Path p = Path::Invalid;
    if (op == 0) p = select_forward(B, H, N, dqk, dv, fmap, dtype);
    if ((op == 3 || op == 4) && check_shape(B, H, N, dqk, dv, fmap, dtype) == LA_OK)
        p = tc_forward_shape(dqk, dv, fmap, dtype) ? Path::FwdTc : Path::FwdSimt;
    if (p == Path::FwdTc) {
        int P, cps, nc;
        tc_segments(B, H, N, &P, &cps, &nc);
        const char *nm = P > 1 ? "fwd_tc_kernel<segment states>,fwd_tc_kernel" : "fwd_tc_kernel";
        if (buf && buflen) {
            strncpy(buf, nm, buflen - 1);
            buf[buflen - 1] = 0;
        }
        return P > 1 ? 2 : 1;
    }
    else if (op == 1 || op == 5) p = select_backward(B, H, N, dqk, dv, fmap, dtype);
    if (p == Path::BwdTc) {
        int P, cps, nc;
        tc_segments(B, H, N, &P, &cps, &nc);
        const bool g = op == 5, tay = bwd_tc_kind(dqk, dv, fmap, dtype) == 3;
        const char *nm =
            P == 1 ? (g ? "bwd_dq_kernel,bwd_dkdv_kernel,bwd_dg_kernel" : "bwd_dq_kernel,bwd_dkdv_kernel")
            : tay  ? (g ? "bwd_sstate_kernel,bwd_dq_kernel,bwd_rstate_kernel,bwd_dkdv_kernel,bwd_dg_kernel"
                        : "bwd_sstate_kernel,bwd_dq_kernel,bwd_rstate_kernel,bwd_dkdv_kernel")
                   : (g ? "bwd_sstate3_kernel,bwd_dq_kernel,bwd_rstate3_kernel,bwd_dkdv_kernel,bwd_dg_kernel"
                        : "bwd_sstate3_kernel,bwd_dq_kernel,bwd_rstate3_kernel,bwd_dkdv_kernel");
        if (buf && buflen) {
            strncpy(buf, nm, buflen - 1);
            buf[buflen - 1] = 0;
        }
        return (P > 1 ? 4 : 2) + (g ? 1 : 0);
    }
    else if (op == 2) p = select_decode(B, H, dqk, dv, fmap, dtype);
    const char *names[8];
    const int n = path_kernels(p, names);
    if (buf && buflen) {
        size_t used = 0;
        buf[0] = 0;
        for (int i = 0; i < n; ++i) {
            const size_t len = strlen(names[i]);
            if (used + len + (i ? 1 : 0) + 1 > buflen) break;
            if (i) buf[used++] = ',';
            memcpy(buf + used, names[i], len);
            used += len;
            buf[used] = 0;
        }
    }
    return n;
}

#ifdef LA_TIMELINE
// Profiling builds only: copy the block-0 role timeline of the last forward.
LA_API int la_debug_timeline_split(long long *events, long long *blocks)
{
    return cudaMemcpyFromSymbol(events, g_tl_split, sizeof(g_tl_split)) == cudaSuccess &&
                   cudaMemcpyFromSymbol(blocks, g_tl_blocks, sizeof(g_tl_blocks)) == cudaSuccess
               ? 0
               : 1;
}
#endif

la_status la_get_device_status(void *stream)
{
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return LA_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_status, sizeof(word)) != cudaSuccess) return LA_ERR_CUDA;
    if (word && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return LA_ERR_CUDA;
    if (word & kStatusTimeout) return LA_ERR_TIMEOUT;
    if (word & kStatusCheck) return LA_ERR_DEVICE_CHECK;
    return LA_OK;
}

la_status la_selftest_bounded_wait(unsigned int wait_us, void *stream)
{
    if (wait_us < 1 || wait_us > 2000000u) return LA_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)wait_us * 1000ull);
    return launch_status();
}

}  // extern "C"
