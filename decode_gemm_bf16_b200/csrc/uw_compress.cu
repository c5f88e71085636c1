// uw_compress.cu -- load-time kernels of the compressor.
//
// "Cloudflare推出Unweight無損壓縮系統" (easyvibecoding.app), §BF16權重壓縮原理:
// each BF16 weight = sign(1) | exponent(8) | mantissa(7); the exponent byte is
// replaced by a palette index (16 most frequent exponents) that is Huffman
// coded; a 64-weight group holding a rarer exponent is kept verbatim.
// §四種執行管道 ("模型載入時預轉"): the palette form is produced once at load.
//
// The host side (uw_host.cpp) runs: histogram -> palette (host) ->
// verbatim flags + symbol counts -> code (host) -> segment bit counts ->
// offsets (host) -> planes, verbatim store, transposed flags, encode.
#include "uw_internal.h"

namespace uw {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t exp_of(uint32_t bf16) { return (bf16 >> 7) & 0xFFu; }
__device__ __forceinline__ uint32_t sm_of(uint32_t bf16) {
    return ((bf16 >> 8) & 0x80u) | (bf16 & 0x7Fu);
}

struct Table256 { uint8_t v[256]; };
struct Table16 { uint8_t v[16]; };
struct Code16 { uint32_t code[16]; uint8_t len[16]; };

// ---- exponent histogram: smem-privatised 256 bins, 8 weights per load.
__global__ void __launch_bounds__(kThreads) k_histogram(const uint4* __restrict__ W, int64_t n8,
                                                        uint32_t* __restrict__ hist) {
    __shared__ uint32_t h[256];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) h[i] = 0;
    __syncthreads();
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
         i += (int64_t)gridDim.x * blockDim.x) {
        uint4 v = W[i];
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            atomicAdd(&h[exp_of(w[j] & 0xFFFFu)], 1u);
            atomicAdd(&h[exp_of(w[j] >> 16)], 1u);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
        if (h[i]) atomicAdd(&hist[i], h[i]);
}

// ---- verbatim flags and symbol frequencies.  One warp per 32 groups; a
// group (64 weights) is read as 32 lanes x 2 weights.
__global__ void __launch_bounds__(kThreads) k_verbatim_freq(const uint32_t* __restrict__ W2,
                                                            int64_t G, Table256 inv_t,
                                                            uint32_t* __restrict__ vbits,
                                                            uint32_t* __restrict__ freq) {
    __shared__ uint8_t inv[256];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) inv[i] = inv_t.v[i];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    uint32_t cnt[16];
#pragma unroll
    for (int v = 0; v < 16; v++) cnt[v] = 0;
    for (int64_t wd = warp; wd * 32 < G; wd += nwarps) {
        uint32_t word = 0;
        for (int j = 0; j < 32; j++) {
            int64_t g = wd * 32 + j;
            if (g >= G) break;
            uint32_t pair = W2[g * 32 + lane];
            uint32_t s0 = inv[exp_of(pair & 0xFFFFu)], s1 = inv[exp_of(pair >> 16)];
            bool verb = __any_sync(0xFFFFFFFFu, s0 == 0xFFu || s1 == 0xFFu);
            if (verb) { s0 = 0; s1 = 0; word |= 1u << j; }
#pragma unroll
            for (int v = 0; v < 16; v++)
                cnt[v] += __popc(__ballot_sync(0xFFFFFFFFu, s0 == (uint32_t)v)) +
                          __popc(__ballot_sync(0xFFFFFFFFu, s1 == (uint32_t)v));
        }
        if (lane == 0) vbits[wd] = word;
    }
    if (lane == 0) {
#pragma unroll
        for (int v = 0; v < 16; v++)
            if (cnt[v]) atomicAdd(&freq[v], cnt[v]);
    }
}

__device__ __forceinline__ bool group_verbatim(const uint32_t* vbits, int64_t g) {
    return (__ldg(&vbits[g >> 5]) >> (g & 31)) & 1u;
}

// ---- bits per 256-symbol segment.  One warp per segment at a time; each
// lane covers 8 weights (one 16-byte load).
__global__ void __launch_bounds__(kThreads) k_segbits(const uint4* __restrict__ W8, int64_t n,
                                                      int64_t nseg, Table256 lenof_t,
                                                      uint8_t len0, const uint32_t* __restrict__ vbits,
                                                      uint32_t* __restrict__ segbits) {
    __shared__ uint8_t lenof[256];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) lenof[i] = lenof_t.v[i];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t j = warp; j < nseg; j += nwarps) {
        int64_t e0 = j * kSeg + lane * 8;
        uint32_t bits = 0;
        if (e0 < n) {
            if (group_verbatim(vbits, e0 / kGroup)) {
                bits = 8u * len0;
            } else {
                uint4 v = W8[e0 / 8];
                uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; q++)
                    bits += lenof[exp_of(w[q] & 0xFFFFu)] + lenof[exp_of(w[q] >> 16)];
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) bits += __shfl_xor_sync(0xFFFFFFFFu, bits, o);
        if (lane == 0) segbits[j] = bits;
    }
}

// ---- sign+mantissa plane and 4-bit index plane.
__global__ void __launch_bounds__(kThreads) k_planes(const uint4* __restrict__ W8, int64_t n8,
                                                     Table256 inv_t, const uint32_t* __restrict__ vbits,
                                                     uint2* __restrict__ sm8, uint32_t* __restrict__ idx8) {
    __shared__ uint8_t inv[256];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) inv[i] = inv_t.v[i];
    __syncthreads();
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
         i += (int64_t)gridDim.x * blockDim.x) {
        uint4 v = W8[i];
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
        bool verb = group_verbatim(vbits, (i * 8) / kGroup);
        uint32_t smw[2] = {0, 0}, ix = 0;
#pragma unroll
        for (int q = 0; q < 4; q++) {
            uint32_t lo = w[q] & 0xFFFFu, hi = w[q] >> 16;
            smw[q >> 1] |= (sm_of(lo) | (sm_of(hi) << 8)) << (16 * (q & 1));
            uint32_t s0 = verb ? 0u : inv[exp_of(lo)], s1 = verb ? 0u : inv[exp_of(hi)];
            ix |= (s0 | (s1 << 4)) << (8 * q);
        }
        sm8[i] = make_uint2(smw[0], smw[1]);
        if (idx8) idx8[i] = ix;
    }
}

// ---- verbatim store: raw exponent bytes of each verbatim group, in group order.
__global__ void __launch_bounds__(kThreads) k_vexp(const uint16_t* __restrict__ W, int64_t G,
                                                   const uint32_t* __restrict__ vbits,
                                                   const uint32_t* __restrict__ vpre,
                                                   uint8_t* __restrict__ vexp) {
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < G;
         g += (int64_t)gridDim.x * blockDim.x) {
        uint32_t word = vbits[g >> 5];
        if (!((word >> (g & 31)) & 1u)) continue;
        int64_t rank = vpre[g >> 5] + __popc(word & ((1u << (g & 31)) - 1u));
        for (int j = 0; j < kGroup; j++) vexp[rank * kGroup + j] = (uint8_t)exp_of(W[g * kGroup + j]);
    }
}

// ---- verbatim flags transposed: word kt*NW + n/32, bit n%32.
__global__ void __launch_bounds__(kThreads) k_vcol(int64_t N, int64_t KG, int64_t NW,
                                                   const uint32_t* __restrict__ vbits,
                                                   uint32_t* __restrict__ vcol) {
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < KG * NW;
         t += (int64_t)gridDim.x * blockDim.x) {
        int64_t kt = t / NW, w = t % NW;
        uint32_t word = 0;
        for (int b = 0; b < 32; b++) {
            int64_t n = w * 32 + b;
            if (n < N && group_verbatim(vbits, n * KG + kt)) word |= 1u << b;
        }
        vcol[t] = word;
    }
}

// ---- Huffman encode.  One lane per 256-symbol segment; its first bit is
// known from the chunk offsets, so segments are independent.  Words shared
// with a neighbouring segment are merged with atomicOr (stream zeroed first).
__global__ void __launch_bounds__(kThreads) k_encode(const uint16_t* __restrict__ W, int64_t n,
                                                     int64_t nseg, Table256 inv_t, Code16 cd,
                                                     const uint32_t* __restrict__ vbits,
                                                     const uint64_t* __restrict__ chunk_off,
                                                     const uint16_t* __restrict__ seg_rel,
                                                     uint32_t* __restrict__ stream) {
    __shared__ uint8_t inv[256];
    __shared__ uint32_t code[16];
    __shared__ uint8_t len[16];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) inv[i] = inv_t.v[i];
    if (threadIdx.x < 16) { code[threadIdx.x] = cd.code[threadIdx.x]; len[threadIdx.x] = cd.len[threadIdx.x]; }
    __syncthreads();
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < nseg;
         j += (int64_t)gridDim.x * blockDim.x) {
        uint64_t p = chunk_off[j / kChunkSegs] + seg_rel[j];
        int64_t wi = (int64_t)(p >> 5);
        uint32_t nb = (uint32_t)(p & 31);   // pending bits in acc (leading zeros)
        uint64_t acc = 0;
        int64_t e_end = min(n, (j + 1) * (int64_t)kSeg);
        for (int64_t e = j * kSeg; e < e_end; e++) {
            uint32_t s = group_verbatim(vbits, e / kGroup) ? 0u : inv[exp_of(W[e])];
            acc = (acc << len[s]) | code[s];
            nb += len[s];
            if (nb >= 32) {
                atomicOr(&stream[wi++], (uint32_t)(acc >> (nb - 32)));
                nb -= 32;
                acc &= (nb ? ((1ull << nb) - 1ull) : 0ull);
            }
        }
        if (nb) atomicOr(&stream[wi], (uint32_t)(acc << (32 - nb)));
    }
}

int grid_for(int64_t work, int per_block) {
    int64_t b = (work + per_block - 1) / per_block;
    int64_t cap = (int64_t)num_sms() * 8;
    if (b > cap) b = cap;
    return (int)(b < 1 ? 1 : b);
}

}  // namespace

size_t compress_scratch_bytes(const Geometry& g) {
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    return al(256 * 4) + al(16 * 4) + al(g.GW * 4) + al(g.nseg * 4);
}

CompressScratch carve_scratch(void* base, const Geometry& g) {
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    uint8_t* p = (uint8_t*)base;
    CompressScratch s;
    s.hist = (uint32_t*)p; p += al(256 * 4);
    s.freq = (uint32_t*)p; p += al(16 * 4);
    s.vbits = (uint32_t*)p; p += al(g.GW * 4);
    s.segbits = (uint32_t*)p;
    return s;
}

cudaError_t launch_histogram(const uint16_t* W, int64_t n, uint32_t* hist, cudaStream_t s) {
    cudaMemsetAsync(hist, 0, 256 * 4, s);
    k_histogram<<<grid_for(n / 8, kThreads), kThreads, 0, s>>>((const uint4*)W, n / 8, hist);
    return cudaGetLastError();
}

cudaError_t launch_verbatim_freq(const uint16_t* W, const Geometry& g, const uint8_t inv[256],
                                 uint32_t* vbits, uint32_t* freq, cudaStream_t s) {
    Table256 t;
    memcpy(t.v, inv, 256);
    cudaMemsetAsync(freq, 0, 16 * 4, s);
    k_verbatim_freq<<<grid_for(g.GW * 32, kThreads), kThreads, 0, s>>>((const uint32_t*)W, g.G, t,
                                                                       vbits, freq);
    return cudaGetLastError();
}

cudaError_t launch_segbits(const uint16_t* W, const Geometry& g, const uint8_t inv[256],
                           const uint32_t* vbits, const uint8_t len[16], uint32_t* segbits,
                           cudaStream_t s) {
    Table256 lenof;
    for (int e = 0; e < 256; e++) lenof.v[e] = inv[e] == 0xFF ? 0 : len[inv[e]];
    k_segbits<<<grid_for(g.nseg * 32, kThreads), kThreads, 0, s>>>((const uint4*)W, g.n, g.nseg,
                                                                    lenof, len[0], vbits, segbits);
    return cudaGetLastError();
}

cudaError_t launch_planes(const uint16_t* W, const Geometry& g, const uint8_t inv[256],
                          const uint32_t* vbits, uint8_t* sm, uint8_t* idx, cudaStream_t s) {
    Table256 t;
    memcpy(t.v, inv, 256);
    k_planes<<<grid_for(g.n / 8, kThreads), kThreads, 0, s>>>((const uint4*)W, g.n / 8, t, vbits,
                                                              (uint2*)sm, (uint32_t*)idx);
    return cudaGetLastError();
}

cudaError_t launch_vexp(const uint16_t* W, const Geometry& g, const uint32_t* vbits,
                        const uint32_t* vpre, uint8_t* vexp, cudaStream_t s) {
    k_vexp<<<grid_for(g.G, kThreads), kThreads, 0, s>>>(W, g.G, vbits, vpre, vexp);
    return cudaGetLastError();
}

cudaError_t launch_vcol(const Geometry& g, const uint32_t* vbits, uint32_t* vcol, cudaStream_t s) {
    k_vcol<<<grid_for(g.KG * g.NW, kThreads), kThreads, 0, s>>>(g.N, g.KG, g.NW, vbits, vcol);
    return cudaGetLastError();
}

cudaError_t launch_encode(const uint16_t* W, const Geometry& g, const uint8_t inv[256],
                          const uint32_t* vbits, const uint8_t len[16], const uint32_t code[16],
                          const uint64_t* chunk_off, const uint16_t* seg_rel, uint32_t* stream,
                          int64_t nwords, cudaStream_t s) {
    Table256 t;
    memcpy(t.v, inv, 256);
    Code16 cd;
    for (int i = 0; i < 16; i++) { cd.code[i] = code[i]; cd.len[i] = len[i]; }
    cudaMemsetAsync(stream, 0, nwords * 4, s);
    k_encode<<<grid_for(g.nseg, kThreads), kThreads, 0, s>>>(W, g.n, g.nseg, t, cd, vbits, chunk_off,
                                                             seg_rel, stream);
    return cudaGetLastError();
}

}  // namespace uw
