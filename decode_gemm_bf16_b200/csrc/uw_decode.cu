// uw_decode.cu -- HBM-to-HBM Huffman decoders of the Unweight format.
//
// "Cloudflare推出Unweight無損壓縮系統" (easyvibecoding.app), §四種執行管道:
//   full decode       -> the original BF16 matrix (writes the most bytes);
//   exponent decode   -> the exponent bytes only (half the traffic);
//   palette transcode -> 4-bit palette indices (a quarter).
// §解壓與運算資源共享 gives the decoder a 16 KB Huffman table in shared
// memory; here that table is a 4096-entry multi-symbol table (12-bit window ->
// up to five symbols).
//
// Work split: a warp owns 32 consecutive 256-symbol segments (8192 weights).
// Phase 1: lane l decodes segment l from its own start bit (chunk offset +
// segment offset) into 32 words of packed nibbles in shared memory (rotated
// by the lane index so that all lanes hit different banks).  The task's
// stream words are first copied into shared memory (asynchronous 16-byte
// copies, issued while the previous task writes its outputs).  Phase 2: the
// warp walks its 8192 outputs in order, maps nibbles to exponents through the
// palette (byte permutes), patches verbatim groups, merges the sign+mantissa
// bytes and stores coalesced 16-byte vectors.
#include "uw_device.cuh"
#include "uw_internal.h"

namespace uw {
namespace {

constexpr int kMaxWarps = 28;                  // warps of a standalone decoder CTA (one CTA per SM)
constexpr int kBesideWarps = 4;                // decoder CTAs that share SMs with the GEMM
constexpr int kTaskElems = 32 * kSeg;          // 8192 weights per warp task
constexpr int kStreamCapW = 768;               // per-warp stream staging, words (3 KB)
constexpr int kStageSmem = 32 * 32 * 4;        // per-warp decoded nibbles
// The standalone decoders (WARPS == 0: the warp count is the launch's) stage
// each task's stream bits in shared memory: the table walk then refills from
// shared memory instead of L1 (gate shape: exponent 47.6 -> 42.7 us, full
// 73.8 -> 66.6 us).  The 4-warp CTAs that run beside a GEMM keep the stream
// in L1 (their shared memory is fixed).
template <int WARPS>
constexpr bool kStaged = WARPS == 0;
constexpr size_t kWarpSmemStaged = kStageSmem + kStreamCapW * 4;
static_assert(kLutSize * 4 + kMaxWarps * kWarpSmemStaged <= 227 * 1024, "decoder smem");
static_assert(kDecodeBesideSmem == kLutSize * 4 + kBesideWarps * kStageSmem, "beside decoder smem");

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
    uint64_t total_bits;
    void* out;
    unsigned long long* band_ready;   // optional: per-band finished-task counters
    unsigned long long epoch;
    int64_t band_tasks;               // tasks per band of 128 rows (= K/64)
};

// Decodes segment `seg` (nsym symbols, a multiple of 64) into `row`: word k of
// the segment (8 nibbles) is stored at row[(k + rot) & 31].
//
// Bit reservoir: a 64-bit `buf` holds the next stream bits, most significant
// first, `nv` of them valid.  A refill adds 32 bits whenever fewer than 32
// are left, so every refill check is followed by two table reads of at most
// 12 bits each with no further check.  One table read decodes up to five
// symbols from the 12-bit window buf >> 52; consuming them is a 64-bit shift.
// The prefetched word `nxt` is the next refill.  Word reads are clamped to the
// stream, so a corrupt stream cannot read outside it; an undecodable window
// still advances (12 bits) and is reported once per segment.  The last read
// may decode past the segment's last symbol (the bits of the next segment or
// the padding); those symbols are never stored.
template <bool SMEM>
__device__ __forceinline__ uint32_t ldw(const uint32_t* sp, int64_t i) {
    if (SMEM) return sp[i];
    return __ldg(sp + i);
}

// `sp` = the stream words (global), or the warp's staged copy of them (SMEM);
// `bitpos` counts from sp[0]; `last` = last readable word index.
template <bool SMEM>
__device__ __forceinline__ void decode_bits(const DecodeParams& p, const uint32_t* lut, const uint32_t* sp0,
                                            int64_t last_word, uint64_t bitpos, int nsym, uint32_t* row, int rot) {
    const int64_t wi = (int64_t)(bitpos >> 5);
    if (wi + 2 > last_word) {
        raise_status(UW_ERR_DEVICE);
        return;
    }
    const uint32_t* __restrict__ sp = sp0 + wi;
    const int64_t room = last_word - wi;
    const uint32_t last = room > 0x7FFFFFFF ? 0x7FFFFFFFu : (uint32_t)room;   // last readable index
    const uint32_t sh = (uint32_t)(bitpos & 31u);
    uint64_t buf = ((uint64_t)ldw<SMEM>(sp, 0) << 32 | (uint64_t)ldw<SMEM>(sp, 1)) << sh;
    int nv = 64 - (int)sh;                          // 33..64 valid bits
    uint32_t nxt = ldw<SMEM>(sp, 2);
    uint32_t idx = 3;
    uint32_t acc = 0, accn = 0, flags = 0;
    int k = 0, kr = rot;
    const int words = nsym >> 3;
    auto refill = [&]() {
        if (nv < 32) {
            buf |= (uint64_t)nxt << (32 - nv);       // shift 1..24
            nv += 32;
            nxt = ldw<SMEM>(sp, min(idx, last));
            idx++;
        }
    };
    // One table read.  A completed word is stored without a branch (lanes
    // complete words at different reads; selects keep the warp converged).
    // A read adds at most 20 bits to fewer than 32, so it completes at most
    // one word.
    auto step = [&]() {
        const uint32_t ent = lut[(uint32_t)(buf >> 52)];
        flags |= ent;
        const uint32_t nb = lut_bits(ent);
        buf <<= nb;
        nv -= (int)nb;
        const uint32_t sy = ent >> kLutSymShift;
        const uint32_t accn2 = accn + lut_nibble_bits(ent);
        acc |= sy << accn;
        const uint32_t fl = accn2 >> 5;                        // a word is complete
        if (fl) row[kr] = acc;
        const uint32_t carry = sy >> ((32u - accn) & 31u);   // used when fl: accn >= 12, shift in [1, 20]
        acc = fl ? carry : acc;
        accn = accn2 & 31u;
        kr = (kr + (int)fl) & 31;
        k += (int)fl;
    };
    // Pairs of reads while at least two words are missing (both stores stay
    // inside the segment), then single reads up to the last word.
    while (k < words - 1) {
        refill();
        step();
        step();
    }
    while (k < words) {
        refill();
        step();
    }
    if (flags & kLutInvalid) raise_status(UW_ERR_DEVICE);
}

__device__ __forceinline__ uint64_t segment_bitpos(const DecodeParams& p, int64_t seg) {
    return seg < p.nseg ? __ldg(&p.chunk_off[seg >> 4]) + __ldg(&p.seg_rel[seg]) : p.total_bits;
}

// Stream words of one warp task, staged into shared memory with 16-byte
// asynchronous copies: [w0a, w0a + nw) with w0a a multiple of 4.  Copies never
// leave the stream section (its allocation is rounded up to 256 bytes).
struct Staging {
    int64_t w0a;
    int nw;
    bool staged;
};

__device__ __forceinline__ Staging stage_stream(const DecodeParams& p, uint64_t first_bit, uint64_t end_bit,
                                                uint32_t* sbuf, int lane) {
    Staging g;
    g.w0a = (int64_t)(first_bit >> 5) & ~int64_t(3);
    int64_t wend = (int64_t)(end_bit >> 5) + 8;            // look-ahead of the bit reservoir
    if (wend > p.nwords) wend = p.nwords;
    wend = (wend + 3) & ~int64_t(3);
    g.nw = (int)(wend - g.w0a);
    g.staged = g.nw <= kStreamCapW;
    if (g.staged) {
        const uint32_t dst = (uint32_t)__cvta_generic_to_shared(sbuf);
        for (int i = lane * 4; i < g.nw; i += 128)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 4u * i), "l"(p.stream + g.w0a + i)
                         : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    return g;
}

template <int MODE, int WARPS>
__global__ void __launch_bounds__(WARPS ? WARPS * 32 : kMaxWarps * 32, WARPS ? 4 : 1) k_decode(const DecodeParams p) {
    constexpr bool STAGED = kStaged<WARPS>;
    const int nwarps = WARPS ? WARPS : (int)(blockDim.x >> 5);
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t* lut = smem;
    uint32_t* stage = smem + kLutSize;
    {
        const uint4* src = reinterpret_cast<const uint4*>(p.lut);
        uint4* dst = reinterpret_cast<uint4*>(lut);
        for (int i = threadIdx.x; i < kLutSize / 4; i += nwarps * 32) dst[i] = __ldg(&src[i]);
    }
    __syncthreads();
    // programmatic stream serialization: the table load above reads only the
    // committed blob; outputs are touched after the previous kernel ends
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* st = stage + warp * ((STAGED ? kWarpSmemStaged : kStageSmem) / 4);
    uint32_t* sbuf = st + 32 * 32;
    const int64_t ntasks = (p.n + kTaskElems - 1) / kTaskElems;
    const uint32_t P0 = p.pal[0], P1 = p.pal[1], P2 = p.pal[2], P3 = p.pal[3];
    const int64_t stride = (int64_t)gridDim.x * nwarps;

    // Staged software pipeline per warp: the stream bits of the
    // next task are copied into shared memory (asynchronously) while this
    // task's outputs are written; the next task's segment offsets load during
    // this task's decode.
    int64_t task = (int64_t)blockIdx.x * nwarps + warp;
    uint64_t bitpos = 0;
    Staging g = {0, 0, false};
    if (STAGED && task < ntasks) {
        bitpos = segment_bitpos(p, task * 32 + lane);
        const uint64_t endb = lane == 31 ? segment_bitpos(p, task * 32 + 32) : 0;
        g = stage_stream(p, __shfl_sync(0xFFFFFFFFu, bitpos, 0), __shfl_sync(0xFFFFFFFFu, endb, 31), sbuf, lane);
    }
    for (; task < ntasks; task += stride) {
        const int64_t base = task * kTaskElems;
        if (MODE == kDecodeFull) {
            // warm L2 with this task's sign+mantissa bytes, read in phase 2
            const int64_t off = base + (int64_t)lane * 256;
            if (off < p.n) {
                asm volatile("prefetch.global.L2 [%0];" ::"l"(p.sm + off));
                asm volatile("prefetch.global.L2 [%0];" ::"l"(p.sm + off + 128));
            }
        }
        const int64_t next = task + stride;
        uint64_t nbit = 0, nend = 0;
        if (STAGED && next < ntasks) {
            nbit = segment_bitpos(p, next * 32 + lane);
            if (lane == 31) nend = segment_bitpos(p, next * 32 + 32);
        }
        if (STAGED) {
            asm volatile("cp.async.wait_all;" ::: "memory");
            __syncwarp();
        }
        // ---- phase 1: one segment per lane
        {
            const int64_t e0 = (task * 32 + lane) * (int64_t)kSeg;
            const int64_t left = p.n - e0;
            const int nsym = left <= 0 ? 0 : (left < kSeg ? (int)left : kSeg);
            if (nsym > 0) {
                if (STAGED && g.staged)
                    decode_bits<true>(p, lut, sbuf, g.nw - 1, bitpos - (uint64_t)g.w0a * 32u, nsym, st + lane * 32, lane);
                else {
                    const int64_t seg = task * 32 + lane;
                    const uint64_t bp = STAGED ? bitpos : __ldg(&p.chunk_off[seg >> 4]) + __ldg(&p.seg_rel[seg]);
                    decode_bits<false>(p, lut, p.stream, p.nwords - 1, bp, nsym, st + lane * 32, lane);
                }
            }
        }
        __syncwarp();
        if (STAGED && next < ntasks)
            g = stage_stream(p, __shfl_sync(0xFFFFFFFFu, nbit, 0), __shfl_sync(0xFFFFFFFFu, nend, 31), sbuf, lane);
        if (STAGED) bitpos = nbit;
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

// ---------------------------------------------------------------------------
// Fused Huffman-decode GEMV / small-batch product: Y[M,N] = X[M,K] . W^T read
// straight from the Huffman form (sign+mantissa plane + stream + verbatim
// store, ~1.34 bytes per weight), with no decoded plane written to HBM.  The
// pages' Hopper design could not keep the 16 KB decode table beside the
// matmul's buffers (§解壓與運算資源共享); here the decode table, the decoded
// nibbles and the activations share one CTA's shared memory with the
// multiply.
//
// Work split, the decoders' own: a warp task is 32 consecutive 256-weight
// segments (8192 weights; whole segments of consecutive rows, since
// K % 256 == 0).  Phase 1: lane l decodes segment l of the task from its own
// start bit into its shared-memory words (the decoder core above), while the
// task's sign+mantissa bytes are requested into L2.  Phase 2: the warp walks
// the task in order, two segments per step (a half warp each, 16 weights a
// lane): sign+mantissa bytes in coalesced 256-byte reads, exponents from the
// palette or the verbatim store, BF16 rebuilt in registers, fused
// multiply-adds with the activations (consecutive 64-byte blocks per lane,
// conflict-free); each lane sums its products over the steps that stay on
// the same rows, then a fixed xor tree over the 16 lanes gives the sums and
// they are added to their rows in order.  A row
// whose segments span several tasks is stored in pieces, and the last task of
// the row to arrive (a tagged counter per row) adds the pieces in order: the
// result depends on the shape only, never on the launch.
// ---------------------------------------------------------------------------
constexpr int kFusedWarps = 8;

struct FusedParams {
    DecodeParams d;
    const uint16_t* X;
    int M;
    int64_t N, K, KG;
    int S;                     // 256-weight segments per row
    int64_t ntasks;            // tasks of 32 segments
    int pmax;                  // pieces per row at most
    float* part;               // [N][pmax][M] pieces of rows that span tasks
    unsigned long long* cnt;   // [N] tagged arrival counters
    unsigned long long epoch;
    void* Y;
    int out_f32;
};

__device__ __forceinline__ void fma_bf16x2(float2& acc, uint32_t w, float x0, float x1) {
    acc.x = fmaf(__uint_as_float(w << 16), x0, acc.x);
    acc.y = fmaf(__uint_as_float(w & 0xFFFF0000u), x1, acc.y);
}

__device__ __forceinline__ void fused_store(const FusedParams& p, int64_t row, int m, float v) {
    if (p.out_f32) reinterpret_cast<float*>(p.Y)[(int64_t)m * p.N + row] = v;
    else {
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        reinterpret_cast<uint16_t*>(p.Y)[(int64_t)m * p.N + row] = *reinterpret_cast<const uint16_t*>(&h);
    }
}

// Row `row`'s sums (racc[m], identical in every lane) for the segments of
// task `task`: the output itself when the row lies inside the task, else a
// piece, and the row's last arriving task adds the pieces.  Warp-uniform.
template <int MB>
__device__ __forceinline__ void fused_flush(const FusedParams& p, int64_t task, int64_t row, const float (&racc)[MB],
                                            int lane) {
    const int64_t s0 = row * p.S, s1 = s0 + p.S;             // the row's segments
    const int64_t t_first = s0 / 32, t_last = (s1 - 1) / 32;
    float v = 0.f;
#pragma unroll
    for (int m = 0; m < MB; m++)
        if (m == lane) v = racc[m];
    if (t_first == t_last) {
        if (lane < p.M) fused_store(p, row, lane, v);
        return;
    }
    const int pieces = (int)(t_last - t_first + 1);
    if (lane < p.M) p.part[(row * p.pmax + (task - t_first)) * p.M + lane] = v;
    __threadfence();
    __syncwarp();
    unsigned c = 0;
    if (lane == 0) c = arrive_counter(p.cnt + row, p.epoch);
    c = __shfl_sync(0xFFFFFFFFu, c, 0);
    if (c == (unsigned)pieces) {
        __threadfence();
        if (lane < p.M) {
            float sum = 0.f;
            for (int q = 0; q < pieces; q++) sum += __ldcg(p.part + (row * p.pmax + q) * p.M + lane);
            fused_store(p, row, lane, sum);
        }
        // a replay of the same captured call reuses its tag: start again from zero
        if (lane == 0) p.cnt[row] = 0ull;
    }
}

// Batch 1-2 (STAGED): the decoders' launch shape -- one CTA per SM with
// as many warps as make every warp's task count equal, each warp's stream
// words staged in shared memory one task ahead.  Batch 4-16: two CTAs of 8
// warps per SM (more registers a thread), the stream read through L1.  The
// activations are read through L1 (all lanes of a half warp read one
// contiguous KB), so shared memory holds only the table, the nibbles and the
// staged stream.
template <int MB, bool STAGED>
__global__ void __launch_bounds__(STAGED ? kMaxWarps * 32 : kFusedWarps * 32, STAGED ? 1 : 2)
    k_fused_huffman(const FusedParams p) {
    const int nwarps = STAGED ? (int)(blockDim.x >> 5) : kFusedWarps;
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t* lut = smem;
    uint32_t* stage = smem + kLutSize;
    {
        const uint4* src = reinterpret_cast<const uint4*>(p.d.lut);
        uint4* dst = reinterpret_cast<uint4*>(lut);
        for (int i = threadIdx.x; i < kLutSize / 4; i += nwarps * 32) dst[i] = __ldg(&src[i]);
    }
    // programmatic stream serialization: the table comes from the committed
    // blob; activations, pieces and outputs after the previous kernel
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* st = stage + warp * ((STAGED ? kWarpSmemStaged : kStageSmem) / 4);
    uint32_t* sbuf = st + 32 * 32;
    const uint32_t P0 = p.d.pal[0], P1 = p.d.pal[1], P2 = p.d.pal[2], P3 = p.d.pal[3];
    const int M = p.M;
    const int half = lane >> 4, hl = lane & 15;
    const int64_t stride = (int64_t)gridDim.x * nwarps;
    int64_t task = (int64_t)blockIdx.x * nwarps + warp;
    uint64_t bitpos = 0;
    Staging g = {0, 0, false};
    if (STAGED && task < p.ntasks) {
        bitpos = segment_bitpos(p.d, task * 32 + lane);
        const uint64_t endb = lane == 31 ? segment_bitpos(p.d, task * 32 + 32) : 0;
        g = stage_stream(p.d, __shfl_sync(0xFFFFFFFFu, bitpos, 0), __shfl_sync(0xFFFFFFFFu, endb, 31), sbuf, lane);
    }
    for (; task < p.ntasks; task += stride) {
        const int64_t base = task * kTaskElems, seg0 = task * 32;
        {
            // the task's sign+mantissa bytes, read in phase 2, into L2 now
            const int64_t off = base + (int64_t)lane * kSeg;
            if (off < p.d.n) {
                asm volatile("prefetch.global.L2 [%0];" ::"l"(p.d.sm + off));
                asm volatile("prefetch.global.L2 [%0];" ::"l"(p.d.sm + off + 128));
            }
        }
        const int64_t next = task + stride;
        uint64_t nbit = 0, nend = 0;
        if (STAGED && next < p.ntasks) {
            nbit = segment_bitpos(p.d, next * 32 + lane);
            if (lane == 31) nend = segment_bitpos(p.d, next * 32 + 32);
        }
        if (STAGED) {
            asm volatile("cp.async.wait_all;" ::: "memory");
            __syncwarp();
        }
        // ---- phase 1: one segment per lane
        {
            const int64_t seg = seg0 + lane;
            if (seg < p.d.nseg) {
                if (STAGED && g.staged)
                    decode_bits<true>(p.d, lut, sbuf, g.nw - 1, bitpos - (uint64_t)g.w0a * 32u, kSeg, st + lane * 32, lane);
                else {
                    const uint64_t bp = STAGED ? bitpos : __ldg(&p.d.chunk_off[seg >> 4]) + __ldg(&p.d.seg_rel[seg]);
                    decode_bits<false>(p.d, lut, p.d.stream, p.d.nwords - 1, bp, kSeg, st + lane * 32, lane);
                }
            }
        }
        __syncwarp();
        if (STAGED && next < p.ntasks)
            g = stage_stream(p.d, __shfl_sync(0xFFFFFFFFu, nbit, 0), __shfl_sync(0xFFFFFFFFu, nend, 31), sbuf, lane);
        if (STAGED) bitpos = nbit;
        // ---- phase 2: two segments per step, 16 weights a lane
        float racc[MB];
#pragma unroll
        for (int m = 0; m < MB; m++) racc[m] = 0.f;
        int64_t rcur = -1;
        // row and segment-within-row of the two segments of the step (segments
        // 2 it and 2 it + 1 of the task), advanced by two segments per step
        const int64_t row0 = seg0 / p.S;
        const int jr0 = (int)(seg0 - row0 * p.S);
        int64_t rw[2] = {row0, row0};
        int jw[2] = {jr0, jr0 + 1};
        if (jw[1] >= p.S) { jw[1] -= p.S; rw[1]++; }
        // lane partial sums of the steps since the halves' rows last changed
        float lacc[MB];
#pragma unroll
        for (int m = 0; m < MB; m++) lacc[m] = 0.f;
        int it0 = 0;   // first step of the current group
#pragma unroll 1
        for (int it = 0; it < 16; it++) {
            const int j = 2 * it + half;               // segment of the task
            const int k0 = 2 * hl;                     // first nibble word of this lane
            const int64_t gs = seg0 + j;
            float2 pacc[MB];
#pragma unroll
            for (int m = 0; m < MB; m++) pacc[m] = make_float2(0.f, 0.f);
            if (gs < p.d.nseg) {
                const int64_t e = base + (int64_t)j * kSeg + k0 * 8;   // element index
                const int64_t kk = (int64_t)(half ? jw[1] : jw[0]) * kSeg + k0 * 8;   // k within the row
                const uint4 sv = __ldg(reinterpret_cast<const uint4*>(p.d.sm + e));
                uint32_t E[4];
                const int64_t g = e >> 6;
                const uint32_t vw = __ldg(&p.d.vbits[g >> 5]);
                if ((vw >> (g & 31)) & 1u) {
                    const int64_t rank = __ldg(&p.d.vpre[g >> 5]) + __popc(vw & ((1u << (g & 31)) - 1u));
                    const uint4 ev = __ldg(reinterpret_cast<const uint4*>(p.d.vexp + rank * kGroup + (e & 63)));
                    E[0] = ev.x; E[1] = ev.y; E[2] = ev.z; E[3] = ev.w;
                } else {
                    const uint32_t* r = st + j * 32;
                    const uint32_t w0 = r[(k0 + j) & 31], w1 = r[(k0 + 1 + j) & 31];
                    if (p.d.pal_small) {
                        const uint32_t x0 = w0 ^ 0x88888888u, x1 = w1 ^ 0x88888888u;
                        E[0] = palette4_small(w0, x0, P0, P1, P2, P3);
                        E[1] = palette4_small(w0 >> 16, x0 >> 16, P0, P1, P2, P3);
                        E[2] = palette4_small(w1, x1, P0, P1, P2, P3);
                        E[3] = palette4_small(w1 >> 16, x1 >> 16, P0, P1, P2, P3);
                    } else {
                        E[0] = palette4(w0, P0, P1, P2, P3);
                        E[1] = palette4(w0 >> 16, P0, P1, P2, P3);
                        E[2] = palette4(w1, P0, P1, P2, P3);
                        E[3] = palette4(w1 >> 16, P0, P1, P2, P3);
                    }
                }
                const uint32_t S4[4] = {sv.x, sv.y, sv.z, sv.w};
                uint32_t wv[8];
#pragma unroll
                for (int t = 0; t < 4; t++) {
                    const uint2 mm = merge4(E[t], S4[t]);
                    wv[2 * t] = mm.x;
                    wv[2 * t + 1] = mm.y;
                }
#pragma unroll
                for (int m = 0; m < MB; m++) {
                    if (m < M) {
                        const uint4* xp = reinterpret_cast<const uint4*>(p.X + (int64_t)m * p.K + kk);
#pragma unroll
                        for (int t = 0; t < 2; t++) {
                            const uint4 xv = __ldg(xp + t);
                            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                            for (int u = 0; u < 4; u++)
                                fma_bf16x2(pacc[m], wv[4 * t + u], __uint_as_float(xw[u] << 16),
                                           __uint_as_float(xw[u] & 0xFFFF0000u));
                        }
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < MB; m++) lacc[m] += pacc[m].x + pacc[m].y;
            const int64_t r0 = rw[0], r1 = rw[1];
#pragma unroll
            for (int h = 0; h < 2; h++) {
                jw[h] += 2;
                while (jw[h] >= p.S) {
                    jw[h] -= p.S;
                    rw[h]++;
                }
            }
            // at the end of the task or where a half's row changes: the
            // group's sums (a fixed xor tree over each half warp, then both
            // halves' sums to every lane), added to the rows in order
            // (warp-uniform)
            if (it == 15 || seg0 + 2 * (it + 1) >= p.d.nseg || rw[0] != r0 || rw[1] != r1) {
                float s_lo[MB], s_hi[MB];
#pragma unroll
                for (int m = 0; m < MB; m++) {
                    float v = lacc[m];
                    v += __shfl_xor_sync(0xFFFFFFFFu, v, 8);
                    v += __shfl_xor_sync(0xFFFFFFFFu, v, 4);
                    v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
                    v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
                    s_lo[m] = __shfl_sync(0xFFFFFFFFu, v, 0);
                    s_hi[m] = __shfl_sync(0xFFFFFFFFu, v, 16);
                    lacc[m] = 0.f;
                }
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    if (seg0 + 2 * it0 + h >= p.d.nseg) break;   // no segment of this half in the group
                    const int64_t row = h ? r1 : r0;
                    if (row != rcur) {
                        if (rcur >= 0) fused_flush<MB>(p, task, rcur, racc, lane);
                        rcur = row;
#pragma unroll
                        for (int m = 0; m < MB; m++) racc[m] = 0.f;
                    }
#pragma unroll
                    for (int m = 0; m < MB; m++) racc[m] += h ? s_hi[m] : s_lo[m];
                }
                it0 = it + 1;
            }
        }
        if (rcur >= 0) fused_flush<MB>(p, task, rcur, racc, lane);
        __syncwarp();   // phase 1 of the next task overwrites the nibbles
    }
}

}  // namespace

static DecodeParams decode_params(const uw_blob* b, void* out);

static int fused_pmax(int64_t K) { return (int)((K / kSeg + 31) / 32) + 1; }

size_t fused_ws_bytes(int64_t M, int64_t N, int64_t K) {
    if (K % kSeg) return 0;
    const int64_t mc = M < kFusedMaxM ? M : kFusedMaxM;
    const size_t part = (size_t)N * fused_pmax(K) * mc * 4;
    return ((part + 255) & ~size_t(255)) + (((size_t)N * 8 + 255) & ~size_t(255));
}

cudaError_t launch_fused_huffman(const uw_blob* b, const uint16_t* X, int64_t M, void* Y, int out_f32, void* ws,
                                 size_t ws_bytes, cudaStream_t s, uw_status* st) {
    *st = UW_OK;
    if (M == 0) return cudaSuccess;
    if (M > kFusedMaxM || b->geo.K % kSeg) { *st = UW_ERR_UNSUPPORTED; return cudaSuccess; }
    const size_t need = fused_ws_bytes(M, b->geo.N, b->geo.K);
    if (!ws || ws_bytes < need) { *st = UW_ERR_WORKSPACE; return cudaSuccess; }
    FusedParams p;
    p.d = decode_params(b, nullptr);
    p.X = X;
    p.M = (int)M;
    p.N = b->geo.N;
    p.K = b->geo.K;
    p.KG = b->geo.KG;
    p.S = (int)(p.K / kSeg);
    p.ntasks = (b->geo.nseg + 31) / 32;
    p.pmax = fused_pmax(p.K);
    const size_t part = (size_t)p.N * p.pmax * M * 4;
    p.part = (float*)ws;
    p.cnt = (unsigned long long*)((uint8_t*)ws + ((part + 255) & ~size_t(255)));
    p.epoch = gemm_next_epoch();
    p.Y = Y;
    p.out_f32 = out_f32;
    const int mb = M == 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16;
    const bool staged = mb <= 2;
    typedef void (*Kern)(const FusedParams);
    Kern kern = mb == 1 ? k_fused_huffman<1, true> : mb == 2 ? k_fused_huffman<2, true> : mb == 4 ? k_fused_huffman<4, false>
              : mb == 8 ? k_fused_huffman<8, false> : k_fused_huffman<16, false>;
    // batch 1-2: one CTA per SM, warps as for the decoders; else two CTAs of
    // 8 warps per SM (every task resident at once when possible, otherwise
    // CTAs loop)
    int grid = 0, warps = kFusedWarps;
    if (staged) {
        decode_grid(p.ntasks, 0, &grid, &warps);
    } else {
        int64_t g = (p.ntasks + kFusedWarps - 1) / kFusedWarps;
        if (g > (int64_t)num_sms() * 2) g = (int64_t)num_sms() * 2;
        grid = (int)g;
    }
    const size_t smem = (size_t)kLutSize * 4 + (size_t)warps * (staged ? kWarpSmemStaged : kStageSmem);
    const size_t smem_max = staged ? (size_t)kLutSize * 4 + (size_t)kMaxWarps * kWarpSmemStaged : smem;
    static bool attr_set[5][64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const int mi = mb == 1 ? 0 : mb == 2 ? 1 : mb == 4 ? 2 : mb == 8 ? 3 : 4;
    if (!attr_set[mi][dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max);
        // the largest shared-memory carveout: the CTAs above fill it
        if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
        attr_set[mi][dev & 63] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)warps * 32);
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
    p.total_bits = b->total_bits;
    p.out = out;
    p.band_ready = nullptr;
    p.epoch = 0;
    p.band_tasks = b->geo.KG;
    return p;
}

// WARPS == 0: `warps` warps a CTA (staged stream); otherwise WARPS.
template <int WARPS>
static cudaError_t launch_decode_impl(const DecodeParams& p, int mode, int grid, int warps, cudaStream_t s) {
    void (*kern)(const DecodeParams) = mode == kDecodeFull       ? k_decode<kDecodeFull, WARPS>
                                       : mode == kDecodeExponent ? k_decode<kDecodeExponent, WARPS>
                                                                 : k_decode<kDecodeTranscode, WARPS>;
    const size_t per_warp = kStaged<WARPS> ? kWarpSmemStaged : kStageSmem;
    const size_t smem = (size_t)kLutSize * 4 + (size_t)warps * per_warp;
    const size_t smem_max = (size_t)kLutSize * 4 + (size_t)(WARPS ? WARPS : kMaxWarps) * per_warp;
    static bool attr_set[3][64] = {{false}};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[mode][dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max);
        // SMs running decoder CTAs keep the largest shared-memory carveout, so
        // a GEMM CTA can still be placed beside them
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[mode][dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(warps * 32);
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

// One CTA per SM.  A warp's tasks take about the same time, so the launch
// lasts as many task times as the busiest warp has tasks: the fewest rounds
// R that kMaxWarps warps per SM allow, then the fewest warps that still
// finish in R rounds (gate shape: 7168 tasks = 2 rounds of 25 warps on 148
// SMs; CTAs of 8 warps, three per SM, left 64 tasks for a third round on 8
// SMs).  `sms` > 0 overrides the SM count.
void decode_grid(int64_t ntasks, int sms, int* grid, int* warps) {
    if (sms <= 0) sms = num_sms();
    if (ntasks < 1) ntasks = 1;
    const int64_t per_round = (int64_t)sms * kMaxWarps;
    const int64_t rounds = (ntasks + per_round - 1) / per_round;
    int64_t w = (ntasks + (int64_t)sms * rounds - 1) / ((int64_t)sms * rounds);
    if (w > kMaxWarps) w = kMaxWarps;
    if (w < 1) w = 1;
    int64_t g = (ntasks + w * rounds - 1) / (w * rounds);
    if (g > sms) g = sms;
    *grid = (int)g;
    *warps = (int)w;
}

cudaError_t launch_decode(const uw_blob* b, int mode, void* out, int sms, cudaStream_t s) {
    DecodeParams p = decode_params(b, out);
    const int64_t ntasks = (p.n + kTaskElems - 1) / kTaskElems;
    int grid = 0, warps = 0;
    decode_grid(ntasks, sms, &grid, &warps);
    return launch_decode_impl<0>(p, mode, grid, warps, s);
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
    return launch_decode_impl<kBesideWarps>(p, mode, grid, kBesideWarps, s);
}

int decode_status_take() { return unit_status_take(); }

}  // namespace uw
