// uw_decode.cu -- HBM-to-HBM Huffman decoders of the Unweight format.
//
// "Cloudflare推出Unweight無損壓縮系統" (easyvibecoding.app), §四種執行管道:
//   full decode       -> the original BF16 matrix (writes the most bytes);
//   exponent decode   -> the exponent bytes only (half the traffic);
//   palette transcode -> 4-bit palette indices (a quarter).
// §解壓與運算資源共享 gives the decoder a 16 KB Huffman table in shared
// memory; here that table is a 4096-entry multi-symbol table (12-bit window ->
// up to four symbols).
//
// Work split: a warp owns 32 consecutive 256-symbol segments (8192 weights).
// Phase 1: lane l decodes segment l from its own start bit (chunk offset +
// segment offset) into 32 words of packed nibbles in shared memory (rotated
// by the lane index so that all lanes hit different banks).  Phase 2: the
// warp walks its 8192 outputs in order, maps nibbles to exponents through the
// palette (byte permutes), patches verbatim groups, merges the sign+mantissa
// bytes and stores coalesced 16-byte vectors.
#include "uw_device.cuh"
#include "uw_internal.h"

namespace uw {
namespace {

constexpr int kWarps = 8;
constexpr int kBesideWarps = 4;                // decoder CTAs that share SMs with the GEMM
constexpr int kTaskElems = 32 * kSeg;          // 8192 weights per warp task
constexpr size_t kDecodeSmem = kLutSize * 4 + kWarps * 32 * 32 * 4;

struct DecodeParams {
    const uint32_t* stream;
    int64_t nwords;
    const uint64_t* chunk_off;
    const uint16_t* seg_rel;
    const uint32_t* lut;
    const uint8_t* sm;
    const uint32_t* vbits;
    const uint32_t* vpre;
    const uint8_t* vexp;
    uint32_t pal[4];
    int pal_small;   // all palette exponents < 128
    int64_t n;       // weights
    int64_t nseg;
    void* out;
    unsigned long long* band_ready;   // optional: per-band finished-task counters
    unsigned long long epoch;
    int64_t band_tasks;               // tasks per band of 128 rows (= K/64)
};

// Decodes segment `seg` (nsym symbols, a multiple of 64) into `row`: word k of
// the segment (8 nibbles) is stored at row[(k + rot) & 31].
//
// Bit reservoir in two 32-bit registers: `hi` holds the next 32 stream bits
// (all valid whenever the table is read), `lo` the following ones, of which
// the top `nlo` are valid.  One table read decodes up to five symbols from the
// 12-bit window hi >> 20; consuming them is a funnel shift.  When lo runs dry
// the prefetched word `nxt` tops the reservoir up.  Word reads are clamped to
// the stream, so a corrupt stream cannot read outside it; an undecodable
// window still advances (12 bits) and is reported once per segment.
__device__ __forceinline__ void decode_segment(const DecodeParams& p, const uint32_t* lut, int64_t seg, int nsym,
                                               uint32_t* row, int rot) {
    const uint64_t bitpos = __ldg(&p.chunk_off[seg >> 4]) + __ldg(&p.seg_rel[seg]);
    const int64_t wi = (int64_t)(bitpos >> 5);
    if (wi + 2 >= p.nwords) {
        raise_status(UW_ERR_DEVICE);
        return;
    }
    const uint32_t* __restrict__ sp = p.stream + wi;
    const int64_t room = p.nwords - 1 - wi;
    const uint32_t last = room > 0x7FFFFFFF ? 0x7FFFFFFFu : (uint32_t)room;   // last readable index
    const uint32_t sh = (uint32_t)(bitpos & 31u);
    const uint32_t w0 = __ldg(sp), w1 = __ldg(sp + 1);
    uint32_t nxt = __ldg(sp + 2);                   // the bits right after lo's valid ones
    uint32_t hi = __funnelshift_l(w1, w0, sh);      // stream bits [bitpos, bitpos + 32)
    uint32_t lo = w1 << sh;                         // rest of w1: 32 - sh valid bits
    int nlo = 32 - (int)sh;
    uint32_t idx = 3;
    uint32_t acc = 0, accn = 0, flags = 0;
    int k = 0, kr = rot;
    const int words = nsym >> 3;
    while (k < words) {
        const uint32_t ent = lut[hi >> 20];
        flags |= ent;
        const uint32_t nb = lut_bits(ent);
        hi = __funnelshift_l(lo, hi, nb);
        lo <<= nb;
        nlo -= (int)nb;
        const uint32_t sy = ent >> kLutSymShift;
        const uint32_t accn2 = accn + lut_nibble_bits(ent);
        acc |= sy << accn;
        if (nlo < 0) {
            hi |= nxt >> (32 + nlo);
            lo = nxt << (-nlo);
            nlo += 32;
            nxt = __ldg(sp + min(idx, last));
            idx++;
        }
        if (accn2 >= 32u) {
            row[kr] = acc;
            kr = (kr + 1) & 31;
            k++;
            acc = sy >> (32u - accn);     // accn >= 12 here, so the shift is in [1, 20]
            accn = accn2 - 32u;
        } else {
            accn = accn2;
        }
    }
    if (flags & kLutInvalid) raise_status(UW_ERR_DEVICE);
}

template <int MODE, int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 4) k_decode(const DecodeParams p) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t* lut = smem;
    uint32_t* stage = smem + kLutSize;
    {
        const uint4* src = reinterpret_cast<const uint4*>(p.lut);
        uint4* dst = reinterpret_cast<uint4*>(lut);
        for (int i = threadIdx.x; i < kLutSize / 4; i += WARPS * 32) dst[i] = __ldg(&src[i]);
    }
    __syncthreads();
    // programmatic stream serialization: the table load above reads only the
    // committed blob; outputs are touched after the previous kernel ends
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* st = stage + warp * 1024;
    const int64_t ntasks = (p.n + kTaskElems - 1) / kTaskElems;
    const uint32_t P0 = p.pal[0], P1 = p.pal[1], P2 = p.pal[2], P3 = p.pal[3];

    for (int64_t task = (int64_t)blockIdx.x * WARPS + warp; task < ntasks;
         task += (int64_t)gridDim.x * WARPS) {
        const int64_t base = task * kTaskElems;
        if (MODE == kDecodeFull) {
            // warm L2 with this task's sign+mantissa bytes, read in phase 2
            const int64_t off = base + (int64_t)lane * 256;
            if (off < p.n) {
                asm volatile("prefetch.global.L2 [%0];" ::"l"(p.sm + off));
                asm volatile("prefetch.global.L2 [%0];" ::"l"(p.sm + off + 128));
            }
        }
        // ---- phase 1: one segment per lane
        {
            int64_t seg = task * 32 + lane;
            int64_t e0 = seg * kSeg;
            int64_t left = p.n - e0;
            int nsym = left <= 0 ? 0 : (left < kSeg ? (int)left : kSeg);
            if (nsym > 0) decode_segment(p, lut, seg, nsym, st + lane * 32, lane);
        }
        __syncwarp();
        // ---- phase 2: ordered, coalesced output (offsets relative to the task)
        const int64_t left = p.n - base;
        const int lim = left < kTaskElems ? (int)left : kTaskElems;
        if (MODE == kDecodeTranscode) {
            // lane -> segment 4*it + lane/8, words 4*(lane%8) .. +3 (32 nibbles)
            uint4* out = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.out) + (base >> 1));
#pragma unroll 2
            for (int it = 0; it < 8; it++) {
                const int j = 4 * it + (lane >> 3);
                const int k0 = 4 * (lane & 7);
                const int e = j * kSeg + k0 * 8;
                if (e < lim) {
                    const uint32_t* r = st + j * 32;
                    uint4 v;
                    v.x = r[(k0 + 0 + j) & 31];
                    v.y = r[(k0 + 1 + j) & 31];
                    v.z = r[(k0 + 2 + j) & 31];
                    v.w = r[(k0 + 3 + j) & 31];
                    out[e >> 5] = v;
                }
            }
        } else {
            // lane -> segment 2*it + lane/16, words 2*(lane%16), +1 (16 weights)
            const uint32_t* vb = p.vbits + (base >> 11);          // 128 groups per task = 4 words
            const uint8_t* smb = p.sm + base;
#pragma unroll 2
            for (int it = 0; it < 16; it++) {
                const int j = 2 * it + (lane >> 4);
                const int k0 = 2 * (lane & 15);
                const int e = j * kSeg + k0 * 8;
                if (e >= lim) continue;
                const uint32_t* r = st + j * 32;
                const uint32_t w0 = r[(k0 + j) & 31], w1 = r[(k0 + 1 + j) & 31];
                uint4 ex;
                const int g = e >> 6;                               // group within the task
                const uint32_t vw = __ldg(&vb[g >> 5]);
                if ((vw >> (g & 31)) & 1u) {
                    const int64_t gg = (base >> 6) + g;
                    const int64_t rank = __ldg(&p.vpre[gg >> 5]) + __popc(vw & ((1u << (g & 31)) - 1u));
                    ex = __ldg(reinterpret_cast<const uint4*>(p.vexp + rank * kGroup + (e & 63)));
                } else if (p.pal_small) {
                    const uint32_t x0 = w0 ^ 0x88888888u, x1 = w1 ^ 0x88888888u;
                    ex.x = palette4_small(w0, x0, P0, P1, P2, P3);
                    ex.y = palette4_small(w0 >> 16, x0 >> 16, P0, P1, P2, P3);
                    ex.z = palette4_small(w1, x1, P0, P1, P2, P3);
                    ex.w = palette4_small(w1 >> 16, x1 >> 16, P0, P1, P2, P3);
                } else {
                    ex.x = palette4(w0, P0, P1, P2, P3);
                    ex.y = palette4(w0 >> 16, P0, P1, P2, P3);
                    ex.z = palette4(w1, P0, P1, P2, P3);
                    ex.w = palette4(w1 >> 16, P0, P1, P2, P3);
                }
                if (MODE == kDecodeExponent) {
                    reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.out) + base)[e >> 4] = ex;
                } else {
                    const uint4 s = __ldg(reinterpret_cast<const uint4*>(smb + e));
                    const uint2 a = merge4(ex.x, s.x), b = merge4(ex.y, s.y);
                    const uint2 c = merge4(ex.z, s.z), d = merge4(ex.w, s.w);
                    uint4* out = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) + base) + (e >> 3);
                    out[0] = make_uint4(a.x, a.y, b.x, b.y);
                    out[1] = make_uint4(c.x, c.y, d.x, d.y);
                }
            }
        }
        __syncwarp();
        if (p.band_ready) {
            // publish: this task's outputs are written
            __threadfence();
            __syncwarp();
            if (lane == 0) arrive_counter(p.band_ready + task / p.band_tasks, p.epoch);
        }
    }
}

}  // namespace

int decode_ctas_per_sm() { return 4; }

static DecodeParams decode_params(const uw_blob* b, void* out) {
    DecodeParams p;
    p.stream = (const uint32_t*)b->sec(UW_SEC_STREAM);
    p.nwords = b->nwords;
    p.chunk_off = (const uint64_t*)b->sec(UW_SEC_CHUNK_OFF);
    p.seg_rel = (const uint16_t*)b->sec(UW_SEC_SEG_REL);
    p.lut = (const uint32_t*)b->sec(UW_SEC_LUT);
    p.sm = b->sec(UW_SEC_SM);
    p.vbits = (const uint32_t*)b->sec(UW_SEC_VBITS);
    p.vpre = (const uint32_t*)b->sec(UW_SEC_VPRE);
    p.vexp = b->sec(UW_SEC_VEXP);
    for (int i = 0; i < 4; i++)
        p.pal[i] = (uint32_t)b->palette[4 * i] | ((uint32_t)b->palette[4 * i + 1] << 8) |
                   ((uint32_t)b->palette[4 * i + 2] << 16) | ((uint32_t)b->palette[4 * i + 3] << 24);
    p.pal_small = 1;
    for (int i = 0; i < 16; i++)
        if (b->palette[i] >= 128) p.pal_small = 0;
    p.n = b->geo.n;
    p.nseg = b->geo.nseg;
    p.out = out;
    p.band_ready = nullptr;
    p.epoch = 0;
    p.band_tasks = b->geo.KG;
    return p;
}

template <int WARPS>
static cudaError_t launch_decode_impl(const DecodeParams& p, int mode, int grid, size_t smem, cudaStream_t s) {
    void (*kern)(const DecodeParams) = mode == kDecodeFull       ? k_decode<kDecodeFull, WARPS>
                                       : mode == kDecodeExponent ? k_decode<kDecodeExponent, WARPS>
                                                                 : k_decode<kDecodeTranscode, WARPS>;
    static bool attr_set[3][64] = {{false}};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[mode][dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        // SMs running decoder CTAs keep the largest shared-memory carveout, so
        // a GEMM CTA can still be placed beside them
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[mode][dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(WARPS * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_decode(const uw_blob* b, int mode, void* out, int grid_ctas, cudaStream_t s) {
    DecodeParams p = decode_params(b, out);
    const int64_t ntasks = (p.n + kTaskElems - 1) / kTaskElems;
    const int64_t need = (ntasks + kWarps - 1) / kWarps;
    int grid = grid_ctas > 0 ? grid_ctas : num_sms() * decode_ctas_per_sm();
    if (grid > need) grid = (int)need;
    if (grid < 1) grid = 1;
    return launch_decode_impl<kWarps>(p, mode, grid, kDecodeSmem, s);
}

cudaError_t launch_decode_beside(const uw_blob* b, int mode, void* out, int ctas, unsigned long long* band_ready,
                                 unsigned long long epoch, cudaStream_t s) {
    DecodeParams p = decode_params(b, out);
    p.band_ready = band_ready;
    p.epoch = epoch;
    const int64_t ntasks = (p.n + kTaskElems - 1) / kTaskElems;
    const int64_t need = (ntasks + kBesideWarps - 1) / kBesideWarps;
    int grid = ctas > need ? (int)need : ctas;
    if (grid < 1) grid = 1;
    return launch_decode_impl<kBesideWarps>(p, mode, grid, kDecodeBesideSmem, s);
}

int decode_status_take() { return unit_status_take(); }

}  // namespace uw
