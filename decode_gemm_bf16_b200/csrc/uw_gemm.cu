// uw_gemm.cu -- Y[M,N] = X[M,K] . W[N,K]^T on the 5th-generation tensor cores,
// with W either plain BF16 or rebuilt on chip from its compressed form.
//
// "Cloudflare推出Unweight無損壓縮系統" (easyvibecoding.app),
// §重建矩陣乘法核心運作: the reconstructive matmul loads compressed data from
// HBM, rebuilds BF16 in shared memory and feeds the tensor cores directly, so
// the rebuilt weights never go back to HBM.  A producer role stages the
// sign+mantissa bytes, the exponent bytes or palette indices and the
// verbatim flags into a ring of shared-memory buffers with TMA, ahead of the
// consumers; consumers merge exponent and sign+mantissa into BF16 tiles.
// §四種執行管道: exponent source (after the exponent decoder), palette source
// (after the transcoder, or straight from the stored index plane).
//
// B200 design (not the Hopper one of the page):
//   * swap-AB: the weight tile is the MMA's A operand (M = 128 rows of W), the
//     activations are B (N = batch tile MG <= 256), the accumulator lives in
//     tensor memory (TMEM) -- no register-file accumulators, so shared memory
//     holds only the stage ring;
//   * warp roles: warps 0-3 epilogue (TMEM lanes 32w..32w+31), warp 4 TMA
//     producer, warp 5 allocates TMEM and issues tcgen05.mma, warps 6-21
//     rebuild BF16 rows (two groups of eight, alternate stages); the producer
//     and MMA warps walk their loops as whole warps and one elected lane
//     issues;
//   * a stage covers 128 k for batch tiles up to 64 rows (64 k above), so the
//     per-stage barrier, TMA and commit costs are paid once per 128 k;
//   * the rebuilt tile never touches shared memory: each rebuild thread owns
//     one weight row (one TMEM lane) and one or two 32-k pieces of the stage,
//     reads its sign+mantissa and index (or exponent) bytes from TMA tiles
//     staged with a swizzle matching their row length (conflict-free
//     row-per-lane reads), and writes 16 columns of BF16 pairs per piece into
//     tensor memory with tcgen05.st; the MMA reads A from TMEM.  Shared memory
//     then carries 3 bytes per weight (TMA write + one read) instead of 7,
//     and holds no A tiles;
//   * stream-K: the (tile, stage) iterations are split evenly over one CTA
//     per SM (or one CTA per tile when that is cheaper, see launch_gemm);
//     tiles are numbered batch-tile-major, so the CTAs working on the batch
//     tiles of one weight tile do so at about the same time and its planes
//     come from HBM about once (L2 serves the other reads); a
//     tile cut between CTAs is finished by the CTA holding its first k steps,
//     which reaches it last and adds the others' fp32 partial rows in k order
//     (deterministic).  This covers batch 1-1024 and the long-K down
//     projection with the same kernel;
//   * weight planes that come from the committed blob are requested before
//     the wait on the previous kernel (programmatic dependent launch);
//   * every wait is bounded (globaltimer deadline); on expiry the CTA raises
//     UW_ERR_TIMEOUT, drains its own TMA and MMA work, frees TMEM and exits.
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <random>
#include <tuple>
#include <vector>

#include "uw_device.cuh"
#include "uw_internal.h"

namespace uw {
namespace {

constexpr int kBlockN = 128;   // weight rows per tile (MMA M)
constexpr int kBoxK = 64;      // k per TMA box of BF16: one 128-byte swizzle row
constexpr int kEpiWarps = 4;
constexpr int kProdWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kReconWarp0 = 6;
constexpr int kReconWarps = 16;       // two groups of 8, one per stage parity
constexpr int kReconGroupWarps = 8;
constexpr int kMaxStages = 8;
constexpr int kThreadsDense = 6 * 32;
constexpr int kThreadsRecon = (kReconWarp0 + kReconWarps) * 32;
// Per stage of KB k (KB = 64 or 128): BF16 weight tile 128 x KB (dense
// source), sign+mantissa 128 x KB bytes, exponents 128 x KB bytes or palette
// indices 128 x KB/2 bytes, and KB/64 words of 128 verbatim flags.
constexpr uint32_t kTileA64 = kBlockN * kBoxK * 2;       // 16 KB: one 64-k box of BF16 weights
constexpr uint32_t kVSlot = 128;     // shared bytes per verbatim-flag slot (stage, matrix) of the flag ring
constexpr uint32_t kStgBytes = 4096; // output transpose buffers: 1 KB per epilogue warp
constexpr int kEpiBar = 1;           // named barrier of the four epilogue warps

// One weight matrix's planes as a stage sees them: where its TMA tiles sit
// in the stage, its verbatim store and its palette.  A paired call (gate and
// up projections, SwiGLU epilogue) carries two.
struct PlaneSet {
    uint32_t off_sm, off_s2;          // stage offsets: sign+mantissa, exponent/index
    int pal_small;                    // all palette exponents < 128: cheaper lookup
    const uint32_t* vbits;
    const uint32_t* vpre;
    const uint8_t* vexp;
    uint32_t pal[4];
};

struct GemmParams {
    int64_t M, N, K, KG;
    int MG, m_tiles, n_tiles, kt_count, P, stages;
    int nh;               // weight matrices per tile: 1, or 2 (gate, up) with the SwiGLU epilogue
    int acc_w;            // accumulator columns per tile: nh * MG (gate in [0, MG), up in [MG, 2 MG))
    uint32_t total_iters;
    uint32_t stage_bytes, off_a, off_b, tx_bytes;
    uint32_t tx_x;        // rebuilding sources: the stage's X bytes (on their own barrier; tx_bytes = the planes)
    uint32_t tmem_cols;   // TMEM columns allocated (power of two)
    uint32_t a_col0;      // first TMEM column of the rebuilt-A stages (nh * KB/2 columns each)
    PlaneSet ps[2];
    void* Y;
    int out_f32;
    float* partial;                // [2P][MG/4][128][4]: float4 j of row r at (slot*MG/4 + j)*128 + r
    uint32_t vring_off;            // shared offset of the verbatim-flag ring (kVSlot per stage and matrix)
    uint32_t stg_off;              // shared offset of the epilogue warps' transpose buffers (1 KB each)
    int y_vec;                     // outputs leave in 16-byte runs (else element stores)
    // SwiGLU in three launches: the finished accumulators go here instead
    // of Y, per tile as float4 columns of 128 rows (block t at t * MG * 128
    // floats; the stream-K partial layout)
    float* gate_out;
    unsigned long long* flags;     // [2P][128]: call tag once a slot's row is published
    unsigned long long epoch;      // 48-bit tag of this call
    // decoder running beside the GEMM: band b of 128 rows is ready when
    // band_ready[b] shows band_tasks(b) finished decoder tasks of this call
    const unsigned long long* band_ready;
    int64_t band_tasks, ntasks;
    uint64_t timeout_ns;
    int static_sm;                 // sign+mantissa plane and verbatim flags come from the committed blob
    int static_s2;                 // so does the second plane (the stored index plane)
};

// Stream-K split: CTA b owns iterations [iter_begin(b), iter_begin(b+1)) of
// the (tile, k step) sequence.  total * P < 2^32 is checked on the host.
// b <= P and i < total, so every product below is under 2^32.
__host__ __device__ __forceinline__ uint32_t iter_begin(uint32_t b, uint32_t total, uint32_t P) {
    return b * total / P;
}
// CTA that processes iteration i (the last b with iter_begin(b) <= i).
__host__ __device__ __forceinline__ uint32_t iter_owner(uint32_t i, uint32_t total, uint32_t P) {
    return ((i + 1) * P - 1) / total;
}
// Partial-sum slot of CTA b's segment of `tile`: its first segment or its last.
__device__ __forceinline__ uint32_t slot_of(uint32_t b, uint32_t tile, uint32_t total, uint32_t P, uint32_t kt) {
    return 2u * b + ((iter_begin(b, total, P) / kt) == tile ? 0u : 1u);
}

// Position in the stage ring: slot and phase parity of iteration q, advanced
// one iteration at a time (no division in the per-stage loops).
struct RingPos {
    int s = 0;
    uint32_t ph = 0;
    __device__ __forceinline__ void advance(int S) {
        if (++s == S) {
            s = 0;
            ph ^= 1u;
        }
    }
};

struct Segment {
    uint32_t tile;
    int kt0, kt1;
    bool first;   // first segment of this CTA's range
};

// Walks the segments of CTA b: [begin, end) cut at tile boundaries.
struct SegWalker {
    uint32_t it, end, kt_count;
    bool started = false;
    __device__ SegWalker(uint32_t b, const GemmParams& p)
        : it(iter_begin(b, p.total_iters, p.P)), end(iter_begin(b + 1, p.total_iters, p.P)),
          kt_count((uint32_t)p.kt_count) {}
    __device__ bool next(Segment& s) {
        if (it >= end) return false;
        s.tile = it / kt_count;
        s.kt0 = (int)(it - s.tile * kt_count);
        const uint32_t hi = (uint32_t)s.kt0 + (end - it);
        s.kt1 = (int)(hi < kt_count ? hi : kt_count);
        s.first = !started;
        started = true;
        it += (uint32_t)(s.kt1 - s.kt0);
        return true;
    }
};

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Offsets of 16-byte chunk c of row r in TMA tiles stored with a 128-byte,
// 64-byte or 32-byte swizzle (rows of that many bytes): chunk bits XOR
// address bits 7 and up.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }
__device__ __forceinline__ uint32_t sw64_off(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }
__device__ __forceinline__ uint32_t sw32_off(int r, int c) { return r * 32 + ((c ^ ((r >> 2) & 1)) << 4); }

// Rebuilds weight row r = 32q + lane, k = 32j .. 32j+31 of the stage's tile
// (stage of KB k at stage index kt) and writes it to TMEM lane r, columns
// taddr .. +15 (one BF16 pair per column).  Sign+mantissa and exponent
// tiles have rows of KB bytes (swizzle KB), index tiles rows of KB/2 bytes;
// the stage's verbatim flags (KB/64 words of 128 rows) sit at `vflags`.
template <int SRC, int KB>
__device__ __forceinline__ void rebuild_row(const GemmParams& p, const PlaneSet& ps, uint32_t stage, uint32_t vflags,
                                            int64_t n0, int kt, int q, int j, int lane, uint32_t taddr) {
    const int r = 32 * q + lane;
    auto row_off = [&](int c) { return KB == 128 ? sw128_off(r, c) : sw64_off(r, c); };
    const uint32_t SM = stage + ps.off_sm;
    const uint4 s0 = lds128(SM + row_off(2 * j));
    const uint4 s1 = lds128(SM + row_off(2 * j + 1));
    uint32_t E[8];
    if (SRC == kSrcExponent) {
        const uint32_t EX = stage + ps.off_s2;
        const uint4 e0 = lds128(EX + row_off(2 * j));
        const uint4 e1 = lds128(EX + row_off(2 * j + 1));
        E[0] = e0.x; E[1] = e0.y; E[2] = e0.z; E[3] = e0.w;
        E[4] = e1.x; E[5] = e1.y; E[6] = e1.z; E[7] = e1.w;
    } else {
        const int grp = j >> 1;   // 64-weight group within the stage
        const uint32_t vw = lds32(vflags + 16 * grp + 4 * q);
        if ((vw >> lane) & 1u) {
            // verbatim group: raw exponents from the verbatim store
            const int64_t g = (n0 + r) * p.KG + (int64_t)kt * (KB / kGroup) + grp;
            const uint32_t w = __ldg(&ps.vbits[g >> 5]);
            const int64_t rank = __ldg(&ps.vpre[g >> 5]) + __popc(w & ((1u << (g & 31)) - 1u));
            const uint4* src = reinterpret_cast<const uint4*>(ps.vexp + rank * kGroup + 32 * (j & 1));
            const uint4 e0 = __ldg(src), e1 = __ldg(src + 1);
            E[0] = e0.x; E[1] = e0.y; E[2] = e0.z; E[3] = e0.w;
            E[4] = e1.x; E[5] = e1.y; E[6] = e1.z; E[7] = e1.w;
        } else {
            const uint4 ix = lds128(stage + ps.off_s2 + (KB == 128 ? sw64_off(r, j) : sw32_off(r, j)));
            const uint32_t w[4] = {ix.x, ix.y, ix.z, ix.w};
            const uint32_t P0 = ps.pal[0], P1 = ps.pal[1], P2 = ps.pal[2], P3 = ps.pal[3];
            if (ps.pal_small) {
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const uint32_t xs = w[i] ^ 0x88888888u;
                    E[2 * i] = palette4_small(w[i], xs, P0, P1, P2, P3);
                    E[2 * i + 1] = palette4_small(w[i] >> 16, xs >> 16, P0, P1, P2, P3);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    E[2 * i] = palette4(w[i], P0, P1, P2, P3);
                    E[2 * i + 1] = palette4(w[i] >> 16, P0, P1, P2, P3);
                }
            }
        }
    }
    const uint32_t S[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    uint32_t out[16];
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const uint2 m = merge4(E[i], S[i]);
        out[2 * i] = m.x;
        out[2 * i + 1] = m.y;
    }
    tmem_st16(taddr, out);
}

__device__ __forceinline__ uint16_t f2bf(float f) {
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&h);
}

// Y[m0 + i, n] for the 16 fp32 values v[i] (bit patterns) of output row n.
__device__ __forceinline__ void store_y(void* Y, int64_t M, int64_t N, int out_f32, const uint32_t (&v)[16], int64_t n,
                                        int64_t m0) {
    if (n >= N || m0 >= M) return;
    const int mv = M - m0 < 16 ? (int)(M - m0) : 16;
    if (out_f32) {
        float* y = reinterpret_cast<float*>(Y) + m0 * N + n;
#pragma unroll
        for (int i = 0; i < 16; i++, y += N)
            if (i < mv) *y = __uint_as_float(v[i]);
    } else {
        uint16_t* y = reinterpret_cast<uint16_t*>(Y) + m0 * N + n;
#pragma unroll
        for (int i = 0; i < 16; i++, y += N)
            if (i < mv) *y = f2bf(__uint_as_float(v[i]));
    }
}

// SwiGLU of 16 outputs: h = silu(g) * u, silu(g) = g / (1 + e^-g), in fp32
// from the two accumulators (bit patterns in, bit patterns out).
__device__ __forceinline__ void swiglu16(const uint32_t (&g)[16], const uint32_t (&u)[16], uint32_t (&h)[16]) {
#pragma unroll
    for (int i = 0; i < 16; i++) {
        const float gv = __uint_as_float(g[i]);
        h[i] = __float_as_uint(gv / (1.0f + __expf(-gv)) * __uint_as_float(u[i]));
    }
}

// True on all four epilogue warps when `pred` holds on any of their threads
// (a barrier with an OR reduction).
__device__ __forceinline__ bool epi_any(bool pred) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"((uint32_t)pred), "n"(kEpiBar), "n"(4 * 32)
        : "memory");
    return res != 0;
}

// Where finished outputs go.  Thread r of the four epilogue warps holds
// output row n0 + r for 16 consecutive batch rows, so a direct store writes
// 2 bytes per lane at 16 addresses N apart.  Instead each warp transposes
// its 32 rows x 16 batch rows through its own 1 KB of shared memory
// (BF16; fp32 goes 8 batch rows at a time) and writes them back with
// 16-byte stores, four lanes per 64-byte run of a batch row: 2 vector
// stores a lane instead of 16 scalar ones.  Without 16-byte rows (Y
// misaligned, N not a multiple of 8 BF16 / 4 fp32) every thread stores its
// own elements.
struct EpiCtx {
    void* Y;
    int64_t M, N;
    int out_f32, vec;
    uint32_t stg;   // shared address of this warp's 1 KB transpose buffer
};

// Outputs Y[m .. m+15, n0 + r] = v[0..15] (fp32 bit patterns); called by
// whole warps (the same m).
__device__ __forceinline__ void emit16(const EpiCtx& e, const uint32_t (&v)[16], int64_t n0, int r, int64_t m) {
    if (!e.vec) {
        store_y(e.Y, e.M, e.N, e.out_f32, v, n0 + r, m);
        return;
    }
    const int lane = r & 31;
    const int64_t nw = n0 + (r & ~31);   // this warp's first output row
    if (e.out_f32) {
#pragma unroll
        for (int h = 0; h < 2; h++) {
            if (m + 8 * h >= e.M) break;
#pragma unroll
            for (int i = 0; i < 8; i++) sts32(e.stg + (uint32_t)(i * 128 + lane * 4), v[8 * h + i]);
            __syncwarp();
#pragma unroll
            for (int s = 0; s < 2; s++) {
                const int idx = s * 32 + lane, t = idx >> 3, seg = idx & 7;
                const uint4 x = lds128(e.stg + (uint32_t)(t * 128 + seg * 16));
                const int64_t mt = m + 8 * h + t, nn = nw + seg * 4;
                if (mt < e.M && nn < e.N) *reinterpret_cast<uint4*>(reinterpret_cast<float*>(e.Y) + mt * e.N + nn) = x;
            }
            __syncwarp();
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; i++) sts16(e.stg + (uint32_t)(i * 64 + lane * 2), f2bf(__uint_as_float(v[i])));
        __syncwarp();
#pragma unroll
        for (int s = 0; s < 2; s++) {
            const int idx = s * 32 + lane, t = idx >> 2, seg = idx & 3;
            const uint4 x = lds128(e.stg + (uint32_t)(t * 64 + seg * 16));
            const int64_t mt = m + t, nn = nw + seg * 8;
            if (mt < e.M && nn < e.N) *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(e.Y) + mt * e.N + nn) = x;
        }
        __syncwarp();
    }
}

// SwiGLU in three launches (batch tiles above 128 rows): the gate and the up
// launch each store their finished accumulator columns c0 .. c0+15 of tile
// `tile` (this thread's row r) as four float4 in the tile's block --
// coalesced 512-byte warp stores, no conversion -- and k_swiglu_blocks
// combines the two block arrays into H.
struct GinCtx {
    float* out;
    int MG;
};
__device__ __forceinline__ void gin_emit(const GinCtx& gc, const uint32_t (&v)[16], uint32_t tile, int r, int c0) {
    float4* dst = reinterpret_cast<float4*>(gc.out) + ((size_t)tile * (size_t)(gc.MG / 4) + (size_t)(c0 / 4)) * kBlockN +
                  (size_t)r;
#pragma unroll
    for (int q = 0; q < 4; q++)
        dst[(size_t)q * kBlockN] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                               __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
}

// Output of a finished accumulator in TMEM: Y directly, or (paired gate and
// up accumulators) SwiGLU of the two halves, or (GIN) SwiGLU with the gate
// projection read from `gin`.  Accumulator columns of batch rows past M are
// skipped.
template <bool GIN>
__device__ __forceinline__ void write_out(const EpiCtx& e, const GinCtx& gc, uint32_t tile, int MG, int nh, uint32_t trow,
                                          int64_t n0, int r, int64_t m0) {
    for (int c0 = 0; c0 < MG; c0 += 16) {
        if (m0 + c0 >= e.M) break;
        uint32_t v[16];
        tmem_ld16(trow + (uint32_t)c0, v);
        if (nh == 2) {
            uint32_t u[16], h[16];
            tmem_ld16(trow + (uint32_t)(MG + c0), u);
            tmem_wait_ld();
            swiglu16(v, u, h);
            emit16(e, h, n0, r, m0 + c0);
        } else {
            tmem_wait_ld();
            if (GIN)
                gin_emit(gc, v, tile, r, c0);
            else
                emit16(e, v, n0, r, m0 + c0);
        }
    }
}

// Finisher of a split tile: own accumulator (TMEM) + the partial rows of
// CTAs blockIdx.x + 1 .. b_last, added in that (k) order, then Y.  The
// finisher's segment is its CTA's last, so the stage ring is idle: the
// contributors' partials come into it with bulk copies.  A contributor's
// partial is stored as float4 columns of 128 rows, so any block of columns
// of it is one contiguous piece; the columns go in blocks as wide as the
// ring holds for every contributor (and both halves of a paired tile), one
// round of copies per block.  Kept out of line: it runs once per CTA and
// would otherwise set the register budget of the whole kernel.
struct FinArgs {
    const float* partial;
    uint32_t ring, ring_bytes, bar;   // idle stage ring and its mbarrier (shared addresses)
    int AW, MG, nh;                   // accumulator columns (nh * MG), output columns, halves
    uint32_t total, P, kt;
    uint64_t timeout_ns;
};

// Returns the updated finisher barrier phase.
template <bool GIN>
__device__ __noinline__ uint32_t finish_tile(const FinArgs f, const EpiCtx e, const GinCtx gc, uint32_t fin_phase,
                                          uint32_t tile, uint32_t b_last, int64_t n0, int r, int64_t m0, uint32_t trow,
                                          volatile int* abort_flag) {
    const uint32_t nb = b_last - blockIdx.x;   // contributors, in k order after this CTA
    const uint32_t col_bytes = kBlockN * 4u;   // one column of one partial
    const size_t slot_floats = (size_t)f.AW * kBlockN;
    // Block width: the widest multiple of 16 columns that the ring holds for
    // every contributor; when not even 16 do, blocks of 16 columns take the
    // contributors in rounds, and the running sum goes back into TMEM
    // between rounds.
    const uint32_t unit = (uint32_t)f.nh * col_bytes * 16u;
    uint32_t CB = 16, R = f.ring_bytes / unit;
    if (nb * unit <= f.ring_bytes) {
        R = nb;
        CB = (f.ring_bytes / (nb * (uint32_t)f.nh * col_bytes)) & ~15u;
        if (CB > (uint32_t)f.MG) CB = (uint32_t)f.MG;
    }
    for (int cb0 = 0; cb0 < f.MG; cb0 += (int)CB) {
        if (m0 + cb0 >= e.M) break;   // batch rows past M: never output
        const uint32_t cw = (uint32_t)f.MG - (uint32_t)cb0 < CB ? (uint32_t)f.MG - (uint32_t)cb0 : CB;
        const uint32_t piece = cw * col_bytes;
        for (uint32_t i0 = 0; i0 < nb; i0 += R) {
        const uint32_t cnt = nb - i0 < R ? nb - i0 : R;
        const bool last = i0 + cnt == nb;
        named_bar_sync(kEpiBar, 4 * 32);   // the ring is no longer read (previous round, or the MMA)
        if (r == 0) {
            // the tags acquired before (one per row, ordered before this
            // thread by the barrier) cover the partials; the copies read
            // them through the async proxy
            fence_proxy_async_global();
            mbar_arrive_expect_tx(f.bar, cnt * (uint32_t)f.nh * piece);
            for (uint32_t i = 0; i < cnt; i++) {
                const uint32_t sl = slot_of(blockIdx.x + 1 + i0 + i, tile, f.total, f.P, f.kt);
                for (int h = 0; h < f.nh; h++)
                    bulk_load(f.ring + (i * (uint32_t)f.nh + (uint32_t)h) * piece,
                              f.partial + (size_t)sl * slot_floats + (size_t)(h * f.MG + cb0) * kBlockN, piece, f.bar);
            }
        }
        mbar_wait(f.bar, fin_phase, f.timeout_ns, abort_flag);
        fin_phase ^= 1u;
        for (int c0 = cb0; c0 < cb0 + (int)cw; c0 += 16) {
            if (m0 + c0 >= e.M) break;
            uint32_t v[16], u[16];
            tmem_ld16(trow + (uint32_t)c0, v);
            if (f.nh == 2) tmem_ld16(trow + (uint32_t)(f.MG + c0), u);
            tmem_wait_ld();
            for (uint32_t i = 0; i < cnt; i++) {
                const uint32_t base = f.ring + i * (uint32_t)f.nh * piece + (uint32_t)(c0 - cb0) * col_bytes + (uint32_t)r * 16u;
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    const uint4 x = lds128(base + (uint32_t)q * (4u * col_bytes));
                    v[4 * q] = __float_as_uint(__uint_as_float(v[4 * q]) + __uint_as_float(x.x));
                    v[4 * q + 1] = __float_as_uint(__uint_as_float(v[4 * q + 1]) + __uint_as_float(x.y));
                    v[4 * q + 2] = __float_as_uint(__uint_as_float(v[4 * q + 2]) + __uint_as_float(x.z));
                    v[4 * q + 3] = __float_as_uint(__uint_as_float(v[4 * q + 3]) + __uint_as_float(x.w));
                }
                if (f.nh == 2) {
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        const uint4 x = lds128(base + piece + (uint32_t)q * (4u * col_bytes));
                        u[4 * q] = __float_as_uint(__uint_as_float(u[4 * q]) + __uint_as_float(x.x));
                        u[4 * q + 1] = __float_as_uint(__uint_as_float(u[4 * q + 1]) + __uint_as_float(x.y));
                        u[4 * q + 2] = __float_as_uint(__uint_as_float(u[4 * q + 2]) + __uint_as_float(x.z));
                        u[4 * q + 3] = __float_as_uint(__uint_as_float(u[4 * q + 3]) + __uint_as_float(x.w));
                    }
                }
            }
            if (!last) {
                tmem_st16(trow + (uint32_t)c0, v);   // running sum, back into the accumulator
                if (f.nh == 2) tmem_st16(trow + (uint32_t)(f.MG + c0), u);
            } else if (f.nh == 2) {
                uint32_t h[16];
                swiglu16(v, u, h);
                emit16(e, h, n0, r, m0 + c0);
            } else {
                if (GIN)
                    gin_emit(gc, v, tile, r, c0);
                else
                    emit16(e, v, n0, r, m0 + c0);
            }
        }
        if (!last) tmem_wait_st();
        }
    }
    return fin_phase;
}

template <int SRC, int KB, int NH, bool GIN = false>
__device__ __forceinline__ void gemm_body(const CUtensorMap& tm_x, const CUtensorMap& tm_a, const CUtensorMap& tm_s2,
                                          const CUtensorMap& tm_v, const CUtensorMap& tm_a2, const CUtensorMap& tm_s22,
                                          const CUtensorMap& tm_v2, const GemmParams& p) {
    static_assert(KB == 64 || KB == 128, "stage k");
    static_assert(NH == 1 || (NH == 2 && SRC == kSrcPalette), "paired tiles: palette source");
    constexpr int kHalves = KB / kBoxK;   // 64-k boxes of X (and of dense W) per stage
    constexpr bool kRecon = SRC != kSrcDense;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = p.stages;
    uint8_t* ctrl = smem + (size_t)S * p.stage_bytes;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(ctrl);
    uint64_t* recon_bar = full_bar + kMaxStages;
    uint64_t* empty_bar = recon_bar + kMaxStages;
    // rebuilding sources: a stage's X tile lands on its own barrier (the MMA
    // waits for it), so the rebuild waits only for the weight planes
    uint64_t* xfull_bar = empty_bar + kMaxStages;
    uint64_t* accf_bar = xfull_bar + kMaxStages;
    uint64_t* acce_bar = accf_bar + 1;
    uint64_t* final_bar = acce_bar + 1;
    uint64_t* fin_bar = final_bar + 1;   // finisher: contributors' partials landed in the ring
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tmem_cols = p.tmem_cols;
    const CUtensorMap* maps_a[2] = {&tm_a, &tm_a2};
    const CUtensorMap* maps_s2[2] = {&tm_s2, &tm_s22};
    const CUtensorMap* maps_v[2] = {&tm_v, &tm_v2};

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&recon_bar[s]), kReconGroupWarps);
            mbar_init(smem_u32(&empty_bar[s]), 1);
            mbar_init(smem_u32(&xfull_bar[s]), 1);
        }
        mbar_init(smem_u32(accf_bar), 1);
        mbar_init(smem_u32(acce_bar), kEpiWarps);
        mbar_init(smem_u32(final_bar), 1);
        mbar_init(smem_u32(fin_bar), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), tmem_cols);
        tmem_relinquish();
    }
    if (warp == kProdWarp && lane == 0) {
        tma_prefetch_desc(&tm_x);
#pragma unroll
        for (int h = 0; h < NH; h++) {
            tma_prefetch_desc(maps_a[h]);
            if (kRecon) {
                tma_prefetch_desc(maps_s2[h]);
                if (SRC == kSrcPalette) tma_prefetch_desc(maps_v[h]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tacc = *tmem_slot;
    // launched with programmatic stream serialization: the prologue above may
    // overlap the previous kernel; global memory it may write is touched only
    // after it ends (the producer warp waits inside its role, below)
    if (warp != kProdWarp) asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t smem_base = smem_u32(smem);
    const uint32_t vring = smem_base + p.vring_off;

    if (warp == kProdWarp) {
        // ------------------------------------------------------------ TMA producer
        // The whole warp walks the loop (its state stays warp-uniform); one
        // elected lane issues the transfers.
        {
            const bool leader = elect_one();
            // Weight planes read from the committed blob (the sign+mantissa
            // plane and verbatim flags of every rebuilding pipeline, the index
            // plane of the direct-palette one) are not written by any kernel:
            // up to four stages of those tiles are requested before the wait
            // on the previous kernel, so they stream in during that kernel's
            // tail; activations and decoded planes follow the wait.  (More
            // stages compete with the previous kernel's last CTAs for HBM:
            // the down projection at batch 1-8 takes 26.8 us with a whole
            // ring requested early, 26.4 us with four stages; two stages are
            // 1-4 % slower.)
            int npre = 0;
            const int npre_max = S < 4 ? S : 4;
            if (kRecon && p.static_sm && !p.band_ready) {
                SegWalker wk0(blockIdx.x, p);
                Segment sg0;
                while (npre < npre_max && wk0.next(sg0)) {
                    const int n_tile = (int)(sg0.tile % p.n_tiles);
                    for (int kt = sg0.kt0; kt < sg0.kt1 && npre < npre_max; kt++, npre++) {
                        if (!leader) continue;
                        const uint32_t st = smem_base + npre * p.stage_bytes;
                        const uint32_t fb = smem_u32(&full_bar[npre]);
                        mbar_arrive_expect_tx(fb, p.tx_bytes);
#pragma unroll
                        for (int h = 0; h < NH; h++) {
                            const PlaneSet& ps = p.ps[h];
                            tma_load_2d(st + ps.off_sm, maps_a[h], kt * KB, n_tile * kBlockN, fb);
                            if (SRC == kSrcPalette) {
                                tma_load_2d(vring + (uint32_t)(npre * NH + h) * kVSlot, maps_v[h],
                                            n_tile * (kBlockN / 32), kt * kHalves, fb);
                                if (p.static_s2)
                                    tma_load_2d(st + ps.off_s2, maps_s2[h], kt * (KB / 2), n_tile * kBlockN, fb);
                            }
                        }
                    }
                }
            }
            asm volatile("griddepcontrol.wait;" ::: "memory");
            SegWalker wk(blockIdx.x, p);
            Segment sg;
            int64_t q = 0;
            RingPos rp;
            bool ok = true;
            int ready_band = -1;
            while (ok && wk.next(sg)) {
                const int n_tile = (int)(sg.tile % p.n_tiles), m_tile = (int)(sg.tile / p.n_tiles);
                if (p.band_ready && n_tile != ready_band) {
                    // the rows of this tile come from the decoder running beside us
                    const int64_t t0 = (int64_t)n_tile * p.band_tasks;
                    const int64_t left = p.ntasks - t0;
                    const unsigned want = (unsigned)(left < p.band_tasks ? left : p.band_tasks);
                    if (!wait_counter(p.band_ready + n_tile, p.epoch, want, p.timeout_ns, abort_flag)) { ok = false; break; }
                    fence_proxy_async_global();
                    ready_band = n_tile;
                }
                for (int kt = sg.kt0; kt < sg.kt1; kt++, q++, rp.advance(S)) {
                    const int s = rp.s;
                    if (q < npre) {
                        // static tiles already requested: activations and the
                        // decoded plane only
                        if (leader) {
                            const uint32_t st = smem_base + s * p.stage_bytes;
                            const uint32_t fb = smem_u32(&full_bar[s]);
                            const uint32_t xb = smem_u32(&xfull_bar[s]);
                            mbar_arrive_expect_tx(xb, p.tx_x);
#pragma unroll
                            for (int hb = 0; hb < kHalves; hb++)
                                tma_load_2d(st + p.off_b + hb * p.MG * 128, &tm_x, kt * KB + hb * kBoxK, m_tile * p.MG, xb);
                            if (SRC == kSrcExponent)
                                tma_load_2d(st + p.ps[0].off_s2, &tm_s2, kt * KB, n_tile * kBlockN, fb);
                            else if (!p.static_s2)
                                tma_load_2d(st + p.ps[0].off_s2, &tm_s2, kt * (KB / 2), n_tile * kBlockN, fb);
                        }
                        continue;
                    }
                    if (!mbar_wait(smem_u32(&empty_bar[s]), rp.ph ^ 1u, p.timeout_ns, abort_flag)) { ok = false; break; }
                    const uint32_t st = smem_base + s * p.stage_bytes;
                    const uint32_t fb = smem_u32(&full_bar[s]);
                    if (!leader) continue;
                    mbar_arrive_expect_tx(fb, p.tx_bytes);
                    const uint32_t xb = kRecon ? smem_u32(&xfull_bar[s]) : fb;
                    if (kRecon) mbar_arrive_expect_tx(xb, p.tx_x);
                    if (SRC == kSrcDense) {
#pragma unroll
                        for (int hb = 0; hb < kHalves; hb++)
                            tma_load_2d(st + p.off_a + hb * kTileA64, &tm_a, kt * KB + hb * kBoxK, n_tile * kBlockN, fb);
                    } else {
                        // the weight planes first: the rebuild waits for them
#pragma unroll
                        for (int h = 0; h < NH; h++) {
                            const PlaneSet& ps = p.ps[h];
                            tma_load_2d(st + ps.off_sm, maps_a[h], kt * KB, n_tile * kBlockN, fb);
                            if (SRC == kSrcExponent)
                                tma_load_2d(st + ps.off_s2, maps_s2[h], kt * KB, n_tile * kBlockN, fb);
                            else {
                                tma_load_2d(st + ps.off_s2, maps_s2[h], kt * (KB / 2), n_tile * kBlockN, fb);
                                tma_load_2d(vring + (uint32_t)(s * NH + h) * kVSlot, maps_v[h],
                                            n_tile * (kBlockN / 32), kt * kHalves, fb);
                            }
                        }
                    }
#pragma unroll
                    for (int hb = 0; hb < kHalves; hb++)
                        tma_load_2d(st + p.off_b + hb * p.MG * 128, &tm_x, kt * KB + hb * kBoxK, m_tile * p.MG, xb);
                }
            }
            if (!ok) {
                // drain: every load already issued must land before the CTA exits
                for (int64_t qq = q - S < 0 ? 0 : q - S; qq < q; qq++) {
                    mbar_wait(smem_u32(&full_bar[qq % S]), (uint32_t)((qq / S) & 1), p.timeout_ns, nullptr);
                    if (kRecon) mbar_wait(smem_u32(&xfull_bar[qq % S]), (uint32_t)((qq / S) & 1), p.timeout_ns, nullptr);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp walks the loop; one elected lane issues the MMAs
        // and commits.  Paired tiles: the gate rows accumulate into columns
        // [0, MG), the up rows into [MG, 2 MG).
        {
            const bool leader = elect_one();
            const uint32_t idesc = mma_idesc_bf16(kBlockN, p.MG);
            SegWalker wk(blockIdx.x, p);
            Segment sg;
            RingPos rp;
            int j = 0;
            bool ok = true;
            while (ok && wk.next(sg)) {
                if (!mbar_wait(smem_u32(acce_bar), (uint32_t)(j & 1) ^ 1u, p.timeout_ns, abort_flag)) { ok = false; break; }
                tc_fence_after();
                for (int kt = sg.kt0; kt < sg.kt1; kt++, rp.advance(S)) {
                    const int s = rp.s;
                    const uint32_t wb = kRecon ? smem_u32(&recon_bar[s]) : smem_u32(&full_bar[s]);
                    if (!mbar_wait(wb, rp.ph, p.timeout_ns, abort_flag)) { ok = false; break; }
                    if (kRecon && !mbar_wait(smem_u32(&xfull_bar[s]), rp.ph, p.timeout_ns, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_base + s * p.stage_bytes;
                    if (!leader) continue;
#pragma unroll
                    for (int h = 0; h < NH; h++) {
                        // 16 k = 32 bytes further along a swizzled row: +2 in the
                        // descriptor's start-address field (16-byte units)
                        const uint32_t ta0 = tacc + p.a_col0 + (uint32_t)(KB / 2) * (uint32_t)(NH * s + h);
                        const uint32_t dacc = tacc + (uint32_t)(h * p.MG);
#pragma unroll
                        for (int hb = 0; hb < kHalves; hb++) {
                            const uint64_t bd0 = sw128_desc(st + p.off_b + hb * p.MG * 128);
                            const uint64_t ad0 = sw128_desc(st + p.off_a + hb * kTileA64);
#pragma unroll
                            for (int kk = 0; kk < kBoxK / 16; kk++) {
                                const uint32_t acc = (kt > sg.kt0 || hb > 0 || kk > 0) ? 1u : 0u;
                                if (kRecon) {
                                    // A: 8 TMEM columns (16 k) of this stage's rebuilt rows
                                    tc_mma_tmem_a(dacc, ta0 + 8u * (uint32_t)(hb * 4 + kk), bd0 + 2u * kk, idesc, acc);
                                } else {
                                    tc_mma(dacc, ad0 + 2u * kk, bd0 + 2u * kk, idesc, acc);
                                }
                            }
                        }
                    }
                    tc_commit(smem_u32(&empty_bar[s]));
                }
                if (!ok) break;
                if (leader) tc_commit(smem_u32(accf_bar));
                j++;
            }
            // drain the tensor core before TMEM is released
            if (leader) tc_commit(smem_u32(final_bar));
            mbar_wait(smem_u32(final_bar), 0, p.timeout_ns, nullptr);
        }
        __syncwarp();
    } else if (kRecon && warp >= kReconWarp0) {
        // ------------------------------------------------------------ reconstruct
        // warp w may only touch TMEM lanes 32(w%4)..+31.  Two groups of 8
        // warps take the even and the odd ring slots (two stages rebuilt at
        // once; with an odd ring the even group has one slot more); inside a
        // group, two warps per lane quarter, one per half of the stage's k
        // (one or two 32-k pieces each), for each weight matrix of the tile.
        constexpr int kPieces = KB / 64;   // 32-k pieces per warp and stage
        const int rw = warp - kReconWarp0;
        const int group = rw / kReconGroupWarps;
        const int quarter = warp & 3, hh = (rw % kReconGroupWarps) >> 2;
        const uint32_t tlane = tacc + ((uint32_t)(32 * quarter) << 16) + p.a_col0;
        SegWalker wk(blockIdx.x, p);
        Segment sg;
        uint32_t q = 0;
        RingPos rp;
        bool ok = true;
        while (ok && wk.next(sg)) {
            const int64_t n0 = (int64_t)(sg.tile % p.n_tiles) * kBlockN;
            for (int kt = sg.kt0; kt < sg.kt1; kt++, q++, rp.advance(S)) {
                // A ring slot always belongs to the same group (slot parity),
                // so a group's waits on a slot see consecutive mbarrier
                // phases.  Taking alternate iterations instead would, with an
                // odd ring, bring a group back to a slot two phases later,
                // which a parity wait cannot tell from the phase before: a
                // group ahead of the loads would rebuild a slot whose tiles
                // had not landed.
                if ((rp.s & 1) != group) continue;
                const int s = rp.s;
                if (!mbar_wait(smem_u32(&full_bar[s]), rp.ph, p.timeout_ns, abort_flag)) { ok = false; break; }
#pragma unroll
                for (int h = 0; h < NH; h++) {
#pragma unroll
                    for (int pc = 0; pc < kPieces; pc++) {
                        const int j = hh * kPieces + pc;
                        rebuild_row<SRC, KB>(p, p.ps[h], smem_base + (uint32_t)s * p.stage_bytes,
                                             vring + (uint32_t)(s * NH + h) * kVSlot, n0, kt, quarter, j, lane,
                                             tlane + (uint32_t)(KB / 2) * (uint32_t)(NH * s + h) + 16u * (uint32_t)j);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&recon_bar[s]));
            }
        }
    } else if (warp < kEpiWarps) {
        // ------------------------------------------------------------ epilogue
        // A tile cut between CTAs is finished by the CTA holding its first k
        // steps (it reaches the tile last, at the end of its range): the other
        // CTAs publish their fp32 partial rows with a per-row tag, the finisher
        // waits for the tags, adds the partials to its own accumulator in k
        // order and writes Y, then clears the tags for a replay of this call.
        // Partials are stored float4-interleaved across rows, so every warp
        // access covers 512 contiguous bytes and one contributor's partial is
        // one contiguous block.  The four warps decide together to stop on a
        // failed wait: the finisher synchronises them.
        SegWalker wk(blockIdx.x, p);
        Segment sg;
        int j = 0;
        const int r = warp * 32 + lane;
        const uint32_t trow = tacc + ((uint32_t)(warp * 32) << 16);
        const int AW4 = p.acc_w / 4;
        const EpiCtx ec = {p.Y, p.M, p.N, p.out_f32, p.y_vec, smem_base + p.stg_off + (uint32_t)warp * 1024u};
        const GinCtx gc = {p.gate_out, p.MG};
        uint32_t fin_phase = 0;
        while (wk.next(sg)) {
            const int n_tile = (int)(sg.tile % p.n_tiles), m_tile = (int)(sg.tile / p.n_tiles);
            const int64_t n0 = (int64_t)n_tile * kBlockN;
            const int64_t m0 = (int64_t)m_tile * p.MG;
            const bool whole = sg.kt0 == 0 && sg.kt1 == p.kt_count;
            const bool finisher = !whole && sg.kt0 == 0;
            const uint32_t kt = (uint32_t)p.kt_count;
            const uint32_t b_last = finisher ? iter_owner(sg.tile * kt + kt - 1, p.total_iters, p.P) : 0u;
            bool good = true;
            if (finisher)
                for (uint32_t b = blockIdx.x + 1; good && b <= b_last; b++) {
                    const uint32_t sl = slot_of(b, sg.tile, p.total_iters, p.P, kt);
                    good = wait_tag(p.flags + (size_t)sl * kBlockN + r, p.epoch, p.timeout_ns, abort_flag);
                }
            if (good) good = mbar_wait(smem_u32(accf_bar), (uint32_t)(j & 1), p.timeout_ns, abort_flag, 20000);
            if (epi_any(!good)) break;
            tc_fence_after();
            const uint32_t slot = 2u * blockIdx.x + (sg.first ? 0u : 1u);
            if (whole) {
                write_out<GIN>(ec, gc, sg.tile, p.MG, NH, trow, n0, r, m0);
            } else if (!finisher) {
                // publish the partial rows (every accumulator column)
                float4* dst = reinterpret_cast<float4*>(p.partial) + (size_t)slot * AW4 * kBlockN + r;
                for (int c0 = 0; c0 < p.acc_w; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld16(trow + (uint32_t)c0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 4; i++)
                        dst[(size_t)(c0 / 4 + i) * kBlockN] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                                          __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
                }
            } else {
                const FinArgs fa = {p.partial, smem_base, (uint32_t)p.stages * p.stage_bytes, smem_u32(fin_bar),
                                    p.acc_w, p.MG, NH, p.total_iters, (uint32_t)p.P, kt, p.timeout_ns};
                fin_phase = finish_tile<GIN>(fa, ec, gc, fin_phase, sg.tile, b_last, n0, r, m0, trow, abort_flag);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(acce_bar));
            if (!whole && !finisher) st_release_u64(p.flags + (size_t)slot * kBlockN + r, p.epoch);
            if (finisher)
                for (uint32_t b = blockIdx.x + 1; b <= b_last; b++)
                    p.flags[(size_t)slot_of(b, sg.tile, p.total_iters, p.P, kt) * kBlockN + r] = 0ull;
            j++;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) raise_status(UW_ERR_TIMEOUT);
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tacc, tmem_cols);
    }
}

// Dense source: 6 warps, registers unconstrained.
template <int KB>
__global__ void __launch_bounds__(kThreadsDense, 1)
    k_gemm_dense(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_a,
                 const __grid_constant__ CUtensorMap tm_s2, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_a2, const __grid_constant__ CUtensorMap tm_s22,
                 const __grid_constant__ CUtensorMap tm_v2, const GemmParams p) {
    gemm_body<kSrcDense, KB, 1>(tm_x, tm_a, tm_s2, tm_v, tm_a2, tm_s22, tm_v2, p);
}

// Rebuilding sources: 22 warps, six of them on two of the four SM
// sub-partitions, whose 16 K registers each allow 80 registers a thread; 72
// when a decoder CTA runs beside the GEMM (that leaves one warp's worth of
// registers per sub-partition for it).
template <int SRC, int KB>
__global__ void __maxnreg__(80)
    k_gemm_recon(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_a,
                 const __grid_constant__ CUtensorMap tm_s2, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_a2, const __grid_constant__ CUtensorMap tm_s22,
                 const __grid_constant__ CUtensorMap tm_v2, const GemmParams p) {
    gemm_body<SRC, KB, 1>(tm_x, tm_a, tm_s2, tm_v, tm_a2, tm_s22, tm_v2, p);
}

template <int SRC, int KB>
__global__ void __maxnreg__(72)
    k_gemm_recon_beside(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_s2, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_a2, const __grid_constant__ CUtensorMap tm_s22,
                        const __grid_constant__ CUtensorMap tm_v2, const GemmParams p) {
    gemm_body<SRC, KB, 1>(tm_x, tm_a, tm_s2, tm_v, tm_a2, tm_s22, tm_v2, p);
}

// Gate and up projections in one launch (direct palette, SwiGLU epilogue):
// each stage carries both matrices' tiles for the same rows and k, each
// tile accumulates into two halves of TMEM.
template <int KB>
__global__ void __maxnreg__(80)
    k_gemm_swiglu(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_a,
                  const __grid_constant__ CUtensorMap tm_s2, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_a2, const __grid_constant__ CUtensorMap tm_s22,
                  const __grid_constant__ CUtensorMap tm_v2, const GemmParams p) {
    gemm_body<kSrcPalette, KB, 2>(tm_x, tm_a, tm_s2, tm_v, tm_a2, tm_s22, tm_v2, p);
}

// SwiGLU in three launches (batch tiles above 128 rows, where a paired tile
// would be capped at 128), direct palette: the gate and the up launch keep
// their accumulators per tile in the workspace.
template <int KB>
__global__ void __maxnreg__(80)
    k_gemm_recon_gin(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_s2, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_a2, const __grid_constant__ CUtensorMap tm_s22,
                     const __grid_constant__ CUtensorMap tm_v2, const GemmParams p) {
    gemm_body<kSrcPalette, KB, 1, true>(tm_x, tm_a, tm_s2, tm_v, tm_a2, tm_s22, tm_v2, p);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)ptr;
    }
    return fn;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, size_t esize, const void* base, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t es[2] = {1, 1};
    (void)esize;
    CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int pick_mg(int64_t M) {
    int64_t mg = (M + 15) / 16 * 16;
    if (mg > 256) mg = 256;
    if (mg < 16) mg = 16;
    return (int)mg;
}

// cudaFuncSetAttribute once per (kernel, device, size): it is not free.
cudaError_t set_smem_attr(const void* fn, int bytes) {
    static std::mutex mu;
    static std::vector<std::tuple<const void*, int, int>> done;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    for (auto& t : done)
        if (std::get<0>(t) == fn && std::get<1>(t) == dev && std::get<2>(t) >= bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e == cudaSuccess) done.emplace_back(fn, dev, bytes);
    return e;
}

// 48-bit call tags: a per-process random base plus a running count.
unsigned long long next_epoch() {
    static std::atomic<unsigned long long> ctr{0};
    static const unsigned long long base = [] {
        std::random_device rd;
        return ((unsigned long long)rd() << 20) ^ (unsigned long long)rd();
    }();
    return (base + ctr.fetch_add(1)) & 0xFFFFFFFFFFFFull;
}

uint64_t timeout_ns() {
    static uint64_t t = 0;
    if (!t) {
        const char* e = getenv("UW_TIMEOUT_MS");
        long ms = e ? atol(e) : 2000;
        if (ms < 10) ms = 10;
        t = (uint64_t)ms * 1000000ull;
    }
    return t;
}

}  // namespace

int gemm_default_grid() { return num_sms(); }

// Batch 1 on a projection with fewer than half as many 128-row tiles as
// GEMM CTAs (every tile would be cut several ways along k) runs the GEMV
// under UW_VARIANT_AUTO; the choice depends only on the shape and options,
// never on the weight source, so the pipelines and the dense baseline keep
// identical summation orders.
bool gemv_serves(const GemmArgs& a) {
    if (a.band_ready) return false;
    if (a.variant == UW_VARIANT_GEMV) return true;
    if (a.variant == UW_VARIANT_TENSOR || a.M != 1) return false;
    const int64_t n_tiles = (a.N + kBlockN - 1) / kBlockN;
    const int64_t P = a.grid > 0 ? a.grid : gemm_default_grid();
    return 2 * n_tiles < P;
}

unsigned long long gemm_next_epoch() { return next_epoch(); }

int gemm_status_take() { return unit_status_take(); }

GemmSplit gemm_split(int64_t M, int64_t N, int64_t K, int grid, int split_k, int nh) {
    GemmSplit g;
    g.MG = pick_mg(M);
    if (nh == 2 && g.MG > 128) g.MG = 128;   // two accumulators must fit TMEM beside the rebuilt-A ring
    // stage k: 128 for small batch tiles (halves the per-stage TMA, barrier
    // and MMA-issue overhead per weight byte), 64 where a stage is already
    // large (batch tiles above 64 rows)
    // (paired tiles keep 64-k stages: two A slots per stage would leave too
    // few 128-k stages in TMEM)
    g.KB = (g.MG <= 64 && K % 128 == 0 && nh == 1) ? 128 : 64;
    g.m_tiles = (int)((M + g.MG - 1) / g.MG);
    g.n_tiles = (int)((N + kBlockN - 1) / kBlockN);
    g.kt = (int)(K / g.KB);
    g.tiles = (int64_t)g.m_tiles * g.n_tiles;
    g.total = g.tiles * g.kt;
    const int sms = gemm_default_grid();
    int64_t P;
    if (split_k > 0) {
        // every tile cut into the same number of k ranges, one CTA each
        const int64_t c = split_k < g.kt ? split_k : g.kt;
        P = g.tiles * c;
        if (c >= 2 && P > sms) g.ok = false;   // finishers would wait on CTAs of a later wave
    } else {
        P = grid > 0 ? grid : sms;
        // Default grid: with batch tiles of 64+ rows and no more output tiles
        // than SMs, every tile is cut into the same whole number of k ranges,
        // one CTA each (one CTA per tile when the tiles number half the SMs
        // or more): each CTA then holds a single segment, instead of a tail
        // and a head whose fix-ups move 32-128 KB of fp32 partials per cut
        // and stall the MMA while they are written.
        if (grid == 0 && g.MG >= 64 && g.tiles <= P) P = g.tiles * (P / g.tiles);
    }
    if (P > g.total) P = g.total;
    if (P < 1) P = 1;
    if (P > 0x7FFFFFFF || g.total * P >= (int64_t(1) << 32)) g.ok = false;
    g.P = (int)P;
    g.fixup = P != g.tiles;
    return g;
}

size_t gemm_ws_bytes(int64_t M, int64_t N, int64_t K, int grid, int split_k, int nh) {
    const GemmSplit g = gemm_split(M, N, K, grid, split_k, nh);
    if (!g.fixup) return 256;
    size_t part = (size_t)2 * g.P * nh * g.MG * kBlockN * 4;
    size_t flags = (size_t)2 * g.P * kBlockN * 8;
    return ((part + 255) & ~size_t(255)) + ((flags + 255) & ~size_t(255));
}

static void set_planes(PlaneSet& ps, const uint8_t* palette, const uint32_t* vbits, const uint32_t* vpre,
                       const uint8_t* vexp) {
    ps.vbits = vbits;
    ps.vpre = vpre;
    ps.vexp = vexp;
    ps.pal_small = 1;
    for (int i = 0; i < 4; i++) ps.pal[i] = 0;
    if (palette) {
        for (int i = 0; i < 4; i++)
            ps.pal[i] = (uint32_t)palette[4 * i] | ((uint32_t)palette[4 * i + 1] << 8) |
                        ((uint32_t)palette[4 * i + 2] << 16) | ((uint32_t)palette[4 * i + 3] << 24);
        for (int i = 0; i < 16; i++)
            if (palette[i] >= 128) ps.pal_small = 0;
    }
}

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s, uw_status* st) {
    *st = UW_OK;
    if (a.M == 0) return cudaSuccess;
    if (a.variant < UW_VARIANT_AUTO || a.variant > UW_VARIANT_GEMV) { *st = UW_ERR_INVALID_ARG; return cudaSuccess; }
    const int NH = a.pair ? 2 : 1;
    if ((a.pair || a.gate_out) && (a.src != kSrcPalette || a.variant == UW_VARIANT_GEMV || a.band_ready || a.smem_cap > 0)) {
        *st = UW_ERR_UNSUPPORTED;
        return cudaSuccess;
    }
    if (!a.pair && !a.gate_out && gemv_serves(a)) return launch_gemv(a, s, st);
    const GemmSplit sp = gemm_split(a.M, a.N, a.K, a.grid, a.split_k, NH);
    if (!sp.ok) { *st = a.split_k > 0 ? UW_ERR_INVALID_ARG : UW_ERR_SHAPE; return cudaSuccess; }
    GemmParams p{};
    p.M = a.M;
    p.N = a.N;
    p.K = a.K;
    p.KG = a.K / kGroup;
    p.MG = sp.MG;
    p.nh = NH;
    p.acc_w = NH * sp.MG;
    const int KB = sp.KB;
    p.m_tiles = sp.m_tiles;
    p.n_tiles = sp.n_tiles;
    p.kt_count = sp.kt;
    const int P = sp.P;
    p.total_iters = (uint32_t)sp.total;
    p.P = P;
    set_planes(p.ps[0], a.palette, a.vbits, a.vpre, a.vexp);
    if (a.pair) set_planes(p.ps[1], a.palette2, a.vbits2, a.vpre2, a.vexp2);
    p.Y = a.Y;
    p.out_f32 = a.out_f32;
    p.gate_out = a.gate_out;
    size_t need = gemm_ws_bytes(a.M, a.N, a.K, a.grid, a.split_k, NH);
    if (!a.ws || a.ws_bytes < need) { *st = UW_ERR_WORKSPACE; return cudaSuccess; }
    size_t part = sp.fixup ? (size_t)2 * P * p.acc_w * kBlockN * 4 : 0;
    p.partial = (float*)a.ws;
    p.flags = (unsigned long long*)((uint8_t*)a.ws + ((part + 255) & ~size_t(255)));
    p.epoch = a.epoch ? a.epoch : next_epoch();
    p.band_ready = a.band_ready;
    p.band_tasks = a.band_tasks;
    p.ntasks = a.ntasks;
    p.timeout_ns = timeout_ns();
    p.static_sm = a.static_sm;
    p.static_s2 = a.static_s2;

    // stage layout (all tiles 1024-byte aligned; swizzled TMA destinations)
    const int halves = KB / kBoxK;
    const uint32_t b_bytes = (uint32_t)p.MG * 128 * halves;
    auto al1k = [](uint32_t x) { return (x + 1023u) & ~1023u; };
    uint32_t off = 0;
    p.tx_bytes = a.src == kSrcDense ? b_bytes : 0;
    p.tx_x = b_bytes;
    if (a.src == kSrcDense) {
        p.off_a = 0;
        p.off_b = kTileA64 * halves;
        off = p.off_b + b_bytes;
        p.tx_bytes += kTileA64 * halves;
    } else {
        const uint32_t sm_bytes = kBlockN * KB, idx_bytes = kBlockN * KB / 2, v_bytes = 16 * halves;
        p.off_b = 0;
        off = al1k(b_bytes);
        for (int h = 0; h < NH; h++) {
            PlaneSet& ps = p.ps[h];
            ps.off_sm = off;
            ps.off_s2 = ps.off_sm + sm_bytes;
            if (a.src == kSrcExponent) {
                off = al1k(ps.off_s2 + sm_bytes);
                p.tx_bytes += 2 * sm_bytes;
            } else {
                // (the stage's verbatim flags go to the flag ring)
                off = al1k(ps.off_s2 + idx_bytes);
                p.tx_bytes += sm_bytes + idx_bytes + v_bytes;
            }
        }
    }
    p.stage_bytes = al1k(off);
    // after the ring: barriers (1 KB), the verbatim-flag ring (palette
    // source: kVSlot per stage and matrix), the output transpose buffers;
    // plus 1 KB to align the dynamic shared memory base
    const size_t ctrl = 1024;
    const size_t vring = a.src == kSrcPalette ? al1k((uint32_t)(kMaxStages * NH) * kVSlot) : 0;
    const size_t reserved = 1024 + ctrl + vring + kStgBytes;
    size_t budget = 227 * 1024 - reserved;
    if (a.smem_cap > 0 && (size_t)a.smem_cap < budget + reserved) budget = (size_t)a.smem_cap - reserved;
    int S = (int)(budget / p.stage_bytes);
    if (S > kMaxStages) S = kMaxStages;
    if (a.stages >= 2 && S > a.stages) S = a.stages;
    // TMEM: accumulator columns [0, acc_w); rebuilt-A stages of NH * KB/2
    // columns after it
    uint32_t acc_cols = 32;
    while (acc_cols < (uint32_t)p.acc_w) acc_cols <<= 1;
    if (a.src != kSrcDense) {
        const int s_tmem = (int)((512u - acc_cols) / (uint32_t)(NH * KB / 2));
        if (S > s_tmem) S = s_tmem;

    }
    if (S < 2) { *st = UW_ERR_UNSUPPORTED; return cudaSuccess; }
    p.stages = S;
    // the finisher brings at least 16 columns of one contributor's partial
    // into the idle ring at once
    if (sp.fixup && (size_t)NH * 16 * kBlockN * 4 > (size_t)S * p.stage_bytes) {
        *st = UW_ERR_UNSUPPORTED;
        return cudaSuccess;
    }
    p.vring_off = (uint32_t)((size_t)S * p.stage_bytes + ctrl);
    p.stg_off = (uint32_t)(p.vring_off + vring);
    p.a_col0 = acc_cols;
    uint32_t need_cols = a.src == kSrcDense ? acc_cols : acc_cols + (uint32_t)(NH * KB / 2) * (uint32_t)S;
    p.tmem_cols = 32;
    while (p.tmem_cols < need_cols) p.tmem_cols <<= 1;
    if (p.tmem_cols > 512) { *st = UW_ERR_UNSUPPORTED; return cudaSuccess; }
    size_t smem = (size_t)S * p.stage_bytes + reserved;

    CUtensorMap tx{}, ta{}, ts2{}, tv{}, ta2{}, ts22{}, tv2{};
    bool ok = make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.X, a.K, a.M, a.K * 2, kBoxK, p.MG,
                          CU_TENSOR_MAP_SWIZZLE_128B);
    if (a.src == kSrcDense) {
        ok = ok && make_map_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.W, a.K, a.N, a.K * 2, kBoxK, kBlockN,
                               CU_TENSOR_MAP_SWIZZLE_128B);
        ts2 = ta;
        tv = ta;
    } else {
        // byte planes: rows of KB bytes (swizzle KB), index rows of KB/2 bytes
        const CUtensorMapSwizzle swz = KB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
        const CUtensorMapSwizzle swz_i = KB == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
        const int64_t NW = 4 * ((a.N + 127) / 128);
        for (int h = 0; h < NH; h++) {
            CUtensorMap* m_a = h ? &ta2 : &ta;
            CUtensorMap* m_s2 = h ? &ts22 : &ts2;
            CUtensorMap* m_v = h ? &tv2 : &tv;
            const uint8_t* sm = h ? a.sm2 : a.sm;
            ok = ok && make_map_2d(m_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, sm, a.K, a.N, a.K, KB, kBlockN, swz);
            if (a.src == kSrcExponent) {
                ok = ok && make_map_2d(m_s2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.ex, a.K, a.N, a.K, KB, kBlockN, swz);
                *m_v = *m_s2;
            } else {
                ok = ok && make_map_2d(m_s2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, h ? a.idx2 : a.idx, a.K / 2, a.N, a.K / 2,
                                       KB / 2, kBlockN, swz_i);
                ok = ok && make_map_2d(m_v, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, h ? a.vcol2 : a.vcol, NW, a.K / kGroup,
                                       NW * 4, 4, KB / kGroup, CU_TENSOR_MAP_SWIZZLE_NONE);
            }
        }
    }
    if (NH == 1) {
        ta2 = ta;
        ts22 = ts2;
        tv2 = tv;
    }
    if (!ok) { *st = UW_ERR_CUDA; return cudaSuccess; }
    // Y in 16-byte runs of a batch row where its rows allow (see emit16)
    const size_t ye = a.out_f32 ? 4 : 2;
    p.y_vec = ((uintptr_t)a.Y % 16 == 0) && (a.N * ye) % 16 == 0;

    typedef void (*GemmKernel)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                               const CUtensorMap, const CUtensorMap, const CUtensorMap, const GemmParams);
    GemmKernel kern;
    if (a.gate_out)
        kern = KB == 128 ? k_gemm_recon_gin<128> : k_gemm_recon_gin<64>;
    else if (a.pair)
        kern = KB == 128 ? k_gemm_swiglu<128> : k_gemm_swiglu<64>;
    else if (a.smem_cap > 0 && a.src != kSrcDense)   // room left for decoder CTAs beside
        kern = KB == 128 ? (a.src == kSrcExponent ? k_gemm_recon_beside<kSrcExponent, 128>
                                                  : k_gemm_recon_beside<kSrcPalette, 128>)
                         : (a.src == kSrcExponent ? k_gemm_recon_beside<kSrcExponent, 64>
                                                  : k_gemm_recon_beside<kSrcPalette, 64>);
    else if (KB == 128)
        kern = a.src == kSrcDense      ? k_gemm_dense<128>
               : a.src == kSrcExponent ? k_gemm_recon<kSrcExponent, 128>
                                       : k_gemm_recon<kSrcPalette, 128>;
    else
        kern = a.src == kSrcDense      ? k_gemm_dense<64>
               : a.src == kSrcExponent ? k_gemm_recon<kSrcExponent, 64>
                                       : k_gemm_recon<kSrcPalette, 64>;
    cudaError_t e = set_smem_attr((const void*)kern, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)P);
    cfg.blockDim = dim3(a.src == kSrcDense ? kThreadsDense : kThreadsRecon);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tx, ta, ts2, tv, ta2, ts22, tv2, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// H[m, n] = silu(G) * U from the two launches' tile blocks: thread = one
// float4 column group (4 batch rows) of one output row; a warp covers 32
// consecutive output rows, so its loads are 512 contiguous bytes and its
// stores 32 consecutive outputs of a batch row.
__global__ void __launch_bounds__(256) k_swiglu_blocks(const float4* __restrict__ G, const float4* __restrict__ U, void* H,
                                                       int64_t M, int64_t N, int MG, int n_tiles, int64_t groups,
                                                       int out_f32) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= groups) return;
    const int r = (int)(i % kBlockN);
    const int64_t jt = i / kBlockN;               // (tile, column group)
    const int64_t tile = jt / (MG / 4);
    const int j = (int)(jt % (MG / 4));
    const int64_t n = (tile % n_tiles) * kBlockN + r;
    const int64_t m = (tile / n_tiles) * MG + 4 * j;
    if (n >= N || m >= M) return;
    const float4 g = __ldcs(G + i), u = __ldcs(U + i);
    const float gg[4] = {g.x, g.y, g.z, g.w}, uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; k++) {
        if (m + k >= M) break;
        const float h = gg[k] / (1.0f + __expf(-gg[k])) * uu[k];
        if (out_f32)
            reinterpret_cast<float*>(H)[(m + k) * N + n] = h;
        else
            reinterpret_cast<uint16_t*>(H)[(m + k) * N + n] = f2bf(h);
    }
}

cudaError_t launch_swiglu_blocks(const float* G, const float* U, void* H, int64_t M, int64_t N, int64_t K, int grid,
                                 int split_k, int out_f32, cudaStream_t s) {
    const GemmSplit sp = gemm_split(M, N, K, grid, split_k, 1);
    const int64_t groups = sp.tiles * (sp.MG / 4) * kBlockN;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((groups + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_swiglu_blocks, reinterpret_cast<const float4*>(G),
                                       reinterpret_cast<const float4*>(U), H, M, N, sp.MG, sp.n_tiles, groups, out_f32);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace uw

// ===========================================================================
// Allocation-free variant of the direct-palette GEMM.
//
// Some callers cannot allocate device memory when they call the GEMM: engines
// that reserve all memory at start-up and forbid later allocation, code that
// must not risk the implicit device synchronisation of cudaMalloc/cudaFree,
// and plugins whose host framework owns the allocator.  For them the stream-K
// fix-up scratch (partial sums and per-row arrival tags) lives in the fixed
// array below, compiled into the library: 4 MiB on every GPU that loads the
// library, held until the process exits.  That covers batches up to 16 on a
// 148-SM B200, for any N.
// ===========================================================================
namespace uw {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (the host-side name of the array is not a device address).
void* noalloc_scratch(uw_status* st) {
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        *st = UW_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            *st = UW_ERR_CUDA;
            return nullptr;
        }
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace
}  // namespace uw

extern "C" uw_status uw_gemm_direct_palette_noalloc(const uint16_t* X, int64_t M, const uw_blob* b, void* Y,
                                                    int out_f32, void* stream) {
    using namespace uw;
    if (!b || b->magic != kMagic || !b->committed || M < 0) return UW_ERR_INVALID_ARG;
    if (!(b->forms & UW_FORM_PALETTE)) return UW_ERR_UNSUPPORTED;
    if (M == 0) return UW_OK;
    if (!X || !Y || ((uintptr_t)X & 15) || ((uintptr_t)Y & 15)) return UW_ERR_INVALID_ARG;
    if (gemm_ws_bytes(M, b->geo.N, b->geo.K, 0, 0, 1) > kNoAllocScratchBytes) return UW_ERR_WORKSPACE;
    uw_status st = UW_OK;
    void* scratch = noalloc_scratch(&st);
    if (!scratch) return st;
    GemmArgs a;
    a.src = kSrcPalette;
    a.X = X;
    a.M = M;
    a.N = b->geo.N;
    a.K = b->geo.K;
    a.sm = b->sec(UW_SEC_SM);
    a.idx = b->sec(UW_SEC_IDX);
    a.static_sm = 1;
    a.static_s2 = 1;
    a.vbits = (const uint32_t*)b->sec(UW_SEC_VBITS);
    a.vpre = (const uint32_t*)b->sec(UW_SEC_VPRE);
    a.vexp = b->sec(UW_SEC_VEXP);
    a.vcol = (const uint32_t*)b->sec(UW_SEC_VCOL);
    a.palette = b->palette;
    a.Y = Y;
    a.out_f32 = out_f32 ? 1 : 0;
    a.grid = 0;
    a.ws = scratch;
    a.ws_bytes = kNoAllocScratchBytes;
    cudaError_t e = launch_gemm(a, (cudaStream_t)stream, &st);
    if (st) return st;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return UW_ERR_CUDA;
    }
    return UW_OK;
}
