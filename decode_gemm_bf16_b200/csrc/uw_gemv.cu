// uw_gemv.cu -- y[N] = W[N,K] . x[K] (batch 1) on the CUDA cores, with W
// plain BF16 or rebuilt in registers from its compressed form.  The GEMM
// entry points route batch 1 here when the projection has few 128-row tiles
// (the tensor-core kernel would cut every tile several ways along k).
//
// "Cloudflare推出Unweight無損壓縮系統" (easyvibecoding.app),
// §重建矩陣乘法核心運作 and §四種執行管道: at batch 1 the matmul is a
// matrix-vector product whose cost is the weight bytes read from HBM; the
// reconstruction (exponent merge or palette lookup + merge) happens on chip
// right before the multiply, so the rebuilt BF16 never returns to HBM.
//
// B200 design: a tensor-core tile would spend one 16-wide MMA column per
// batch row and all of its staging machinery on what is a pure streaming
// problem, so small batches use plain coalesced loads instead:
//   * one warp owns whole weight rows (rows_per_warp of them, in order); a
//     step covers 512 consecutive weights of the row, 16 per lane (inside
//     one 64-weight group), so every plane is read in 512-byte (sign+
//     mantissa, exponents) or 256-byte (indices) coalesced warp accesses,
//     streaming (evict-first); BF16 weights take two 16-byte loads a lane;
//   * each warp issues four steps of loads before using them, and 32 warps
//     per SM keep well over the ~45 KB per SM in flight that HBM3e needs at
//     this latency;
//   * the palette lookup is two byte permutes per four weights, verbatim
//     64-weight groups (rare) read their raw exponents from the verbatim
//     store; the merged BF16 pairs widen to fp32 with a shift or a mask;
//   * activations are converted to fp32 once per CTA into shared memory
//     (when they fit) and each lane accumulates its weights in k order with
//     fp32 fused multiply-adds (even and odd weights in two sums), then a
//     butterfly over the 32 lanes sums the row; the order does not depend on
//     the source, so all sources give identical bits.
#include "uw_device.cuh"
#include "uw_internal.h"

namespace uw {
namespace {

constexpr int kGemvWarps = 16;
constexpr int kLaneW = 16;               // weights per lane per step (within one 64-weight group)
constexpr int kStepW = 32 * kLaneW;      // weights per warp step
constexpr size_t kGemvSmemMax = 112 * 1024;   // fp32 activations in shared memory, two CTAs per SM

struct GemvParams {
    const uint16_t* X;
    int64_t M, N, K, KG;
    const uint16_t* W;
    const uint8_t* sm;
    const uint8_t* ex;
    const uint8_t* idx;
    const uint32_t* vbits;
    const uint32_t* vpre;
    const uint8_t* vexp;
    uint32_t pal[4];
    int pal_small;
    void* Y;
    int out_f32;
    int64_t rows_per_warp;
};

// The raw bytes of one lane's 16 weights: BF16 (two 16-byte vectors), or
// sign+mantissa bytes (a) plus exponent bytes (b) or 16 index nibbles (b.x,
// b.y).
struct StepLoad {
    uint4 a, b;
};

template <int SRC>
__device__ __forceinline__ void load_step(const GemvParams& p, int64_t row0, int64_t k, StepLoad& L) {
    if (SRC == kSrcDense) {
        const uint4* w = reinterpret_cast<const uint4*>(p.W + row0 + k);
        L.a = __ldcs(w);
        L.b = __ldcs(w + 1);
    } else {
        L.a = __ldcs(reinterpret_cast<const uint4*>(p.sm + row0 + k));
        if (SRC == kSrcExponent) {
            L.b = __ldcs(reinterpret_cast<const uint4*>(p.ex + row0 + k));
        } else {
            const uint2 ix = __ldcs(reinterpret_cast<const uint2*>(p.idx + ((row0 + k) >> 1)));
            L.b = make_uint4(ix.x, ix.y, 0u, 0u);
        }
    }
}

// Rebuilds the 16 weights as 8 BF16 pairs (element order); g = their group.
template <int SRC>
__device__ __forceinline__ void rebuild_step(const GemvParams& p, int64_t g, int64_t k, const StepLoad& L,
                                             uint32_t (&w)[8]) {
    if (SRC == kSrcDense) {
        w[0] = L.a.x; w[1] = L.a.y; w[2] = L.a.z; w[3] = L.a.w;
        w[4] = L.b.x; w[5] = L.b.y; w[6] = L.b.z; w[7] = L.b.w;
        return;
    }
    uint32_t E[4];
    if (SRC == kSrcExponent) {
        E[0] = L.b.x; E[1] = L.b.y; E[2] = L.b.z; E[3] = L.b.w;
    } else {
        const uint32_t vw = __ldg(&p.vbits[g >> 5]);
        if ((vw >> (g & 31)) & 1u) {
            // verbatim group: raw exponents from the verbatim store
            const int64_t rank = __ldg(&p.vpre[g >> 5]) + __popc(vw & ((1u << (g & 31)) - 1u));
            const uint4 e = __ldg(reinterpret_cast<const uint4*>(p.vexp + rank * kGroup + (k & 63)));
            E[0] = e.x; E[1] = e.y; E[2] = e.z; E[3] = e.w;
        } else {
            const uint32_t P0 = p.pal[0], P1 = p.pal[1], P2 = p.pal[2], P3 = p.pal[3];
            const uint32_t x0 = L.b.x, x1 = L.b.y;
            if (p.pal_small) {
                const uint32_t s0 = x0 ^ 0x88888888u, s1 = x1 ^ 0x88888888u;
                E[0] = palette4_small(x0, s0, P0, P1, P2, P3);
                E[1] = palette4_small(x0 >> 16, s0 >> 16, P0, P1, P2, P3);
                E[2] = palette4_small(x1, s1, P0, P1, P2, P3);
                E[3] = palette4_small(x1 >> 16, s1 >> 16, P0, P1, P2, P3);
            } else {
                E[0] = palette4(x0, P0, P1, P2, P3);
                E[1] = palette4(x0 >> 16, P0, P1, P2, P3);
                E[2] = palette4(x1, P0, P1, P2, P3);
                E[3] = palette4(x1 >> 16, P0, P1, P2, P3);
            }
        }
    }
    const uint32_t S[4] = {L.a.x, L.a.y, L.a.z, L.a.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const uint2 m = merge4(E[j], S[j]);
        w[2 * j] = m.x;
        w[2 * j + 1] = m.y;
    }
}

// Shared-memory position (in 16-byte chunks) of activation chunk c: lane l
// reads chunks 4l .. 4l+3 of a step, and the XOR spreads the eight lanes of
// each access phase over all eight 16-byte bank groups.
__device__ __forceinline__ uint32_t xs_chunk(uint32_t c) { return (c & ~3u) | ((c ^ (c >> 3)) & 3u); }

// acc.(x, y) += (lo, hi BF16 of w as fp32) * (x0, x1): two fp32 fused
// multiply-adds, even and odd weights in separate sums.
__device__ __forceinline__ void fma2(float2& acc, uint32_t w, float x0, float x1) {
    acc.x = fmaf(__uint_as_float(w << 16), x0, acc.x);
    acc.y = fmaf(__uint_as_float(w & 0xFFFF0000u), x1, acc.y);
}

// XS: activations converted once per CTA to fp32 in shared memory; else read
// as BF16 through L1.
template <int SRC, int MB, bool XS>
__global__ void __launch_bounds__(kGemvWarps * 32, 2) k_gemv(const GemvParams p) {
    constexpr int kBatch = MB == 1 ? 4 : 2;   // steps whose loads are in flight together
    extern __shared__ __align__(16) float xs[];
    const int M = (int)p.M;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (XS) {
        // row m of X occupies chunks [m K/4, (m+1) K/4); K/4 is a multiple of 16
        const uint32_t chunks = (uint32_t)(p.M * p.K / 4);
        for (uint32_t c = threadIdx.x; c < chunks; c += blockDim.x) {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(p.X) + c);
            reinterpret_cast<float4*>(xs)[xs_chunk(c)] =
                make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                            __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
        }
        __syncthreads();
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t)blockIdx.x * kGemvWarps + (threadIdx.x >> 5);
    const int64_t n0 = warp * p.rows_per_warp;
    const int64_t n1 = n0 + p.rows_per_warp < p.N ? n0 + p.rows_per_warp : p.N;
    for (int64_t n = n0; n < n1; n++) {
        const int64_t row0 = n * p.K, g0 = n * p.KG;
        float2 acc[MB];
#pragma unroll
        for (int m = 0; m < MB; m++) acc[m] = make_float2(0.f, 0.f);
        for (int64_t kb = 0; kb < p.K; kb += (int64_t)kBatch * kStepW) {
            StepLoad L[kBatch];
#pragma unroll
            for (int s = 0; s < kBatch; s++) {
                const int64_t k = kb + s * kStepW + lane * kLaneW;
                if (k < p.K) load_step<SRC>(p, row0, k, L[s]);
            }
#pragma unroll
            for (int s = 0; s < kBatch; s++) {
                const int64_t k = kb + s * kStepW + lane * kLaneW;
                if (k < p.K) {
                    uint32_t w[8];
                    rebuild_step<SRC>(p, g0 + (k >> 6), k, L[s], w);
#pragma unroll
                    for (int m = 0; m < MB; m++) {
                        if (m < M) {
                            if (XS) {
                                const float4* x4 = reinterpret_cast<const float4*>(xs);
                                const uint32_t c0 = (uint32_t)(((int64_t)m * p.K + k) >> 2);
#pragma unroll
                                for (int q = 0; q < 4; q++) {
                                    const float4 x = x4[xs_chunk(c0 + q)];
                                    fma2(acc[m], w[2 * q], x.x, x.y);
                                    fma2(acc[m], w[2 * q + 1], x.z, x.w);
                                }
                            } else {
                                const uint4* xp = reinterpret_cast<const uint4*>(p.X + (int64_t)m * p.K + k);
#pragma unroll
                                for (int q = 0; q < 2; q++) {
                                    const uint4 x = __ldg(xp + q);
                                    const uint32_t xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                                    for (int i = 0; i < 4; i++)
                                        fma2(acc[m], w[4 * q + i], __uint_as_float(xv[i] << 16),
                                             __uint_as_float(xv[i] & 0xFFFF0000u));
                                }
                            }
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int m = 0; m < MB; m++) {
            float v = acc[m].x + acc[m].y;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
            if (lane == m && m < M) {
                if (p.out_f32) reinterpret_cast<float*>(p.Y)[(int64_t)m * p.N + n] = v;
                else {
                    const __nv_bfloat16 h = __float2bfloat16_rn(v);
                    reinterpret_cast<uint16_t*>(p.Y)[(int64_t)m * p.N + n] = *reinterpret_cast<const uint16_t*>(&h);
                }
            }
        }
    }
}

template <int SRC, bool XS>
static const void* gemv_kernel_xs(int mb) {
    (void)mb;
    return (const void*)k_gemv<SRC, 1, XS>;
}
template <int SRC>
static const void* gemv_kernel(int mb, bool xs) {
    return xs ? gemv_kernel_xs<SRC, true>(mb) : gemv_kernel_xs<SRC, false>(mb);
}

}  // namespace

cudaError_t launch_gemv(const GemmArgs& a, cudaStream_t s, uw_status* st) {
    *st = UW_OK;
    if (a.M == 0) return cudaSuccess;
    if (a.M > kGemvMaxM) { *st = UW_ERR_UNSUPPORTED; return cudaSuccess; }
    GemvParams p{};
    p.X = a.X;
    p.M = a.M;
    p.N = a.N;
    p.K = a.K;
    p.KG = a.K / kGroup;
    p.W = a.W;
    p.sm = a.sm;
    p.ex = a.ex;
    p.idx = a.idx;
    p.vbits = a.vbits;
    p.vpre = a.vpre;
    p.vexp = a.vexp;
    p.pal_small = 1;
    if (a.palette) {
        for (int i = 0; i < 4; i++)
            p.pal[i] = (uint32_t)a.palette[4 * i] | ((uint32_t)a.palette[4 * i + 1] << 8) |
                       ((uint32_t)a.palette[4 * i + 2] << 16) | ((uint32_t)a.palette[4 * i + 3] << 24);
        for (int i = 0; i < 16; i++)
            if (a.palette[i] >= 128) p.pal_small = 0;
    }
    p.Y = a.Y;
    p.out_f32 = a.out_f32;
    // fewest rows per warp such that all warps are resident (32 per SM)
    const int64_t slots = (int64_t)num_sms() * 32;
    p.rows_per_warp = (a.N + slots - 1) / slots;
    if (p.rows_per_warp < 1) p.rows_per_warp = 1;
    const int64_t warps = (a.N + p.rows_per_warp - 1) / p.rows_per_warp;
    const int64_t grid = (warps + kGemvWarps - 1) / kGemvWarps;
    const int mb = a.M == 1 ? 1 : a.M == 2 ? 2 : 4;
    const size_t xbytes = (size_t)a.M * (size_t)a.K * 4;
    const bool xs = xbytes <= kGemvSmemMax;
    const void* kern = a.src == kSrcDense ? gemv_kernel<kSrcDense>(mb, xs)
                       : a.src == kSrcExponent ? gemv_kernel<kSrcExponent>(mb, xs)
                                               : gemv_kernel<kSrcPalette>(mb, xs);
    const size_t smem = xs ? xbytes : 0;
    static bool attr_set[3][3][64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    bool& done = attr_set[a.src][mb >> 1][dev & 63];
    if (xs && !done) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemvSmemMax);
        if (e != cudaSuccess) return e;
        done = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kGemvWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&p};
    cudaError_t e = cudaLaunchKernelExC(&cfg, kern, args);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace uw
