// uw_internal.h -- host-side state shared by the translation units of
// libunweight.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "../../include/unweight.h"

namespace uw {

constexpr int kGroup = 64;        // weights per verbatim decision
constexpr int kPalette = 16;      // palette entries
constexpr int kSeg = 256;         // symbols per decode segment
constexpr int kChunkSegs = 16;    // segments per chunk offset
constexpr int kLmax = 12;         // longest Huffman code, bits
constexpr int kLutSize = 1 << kLmax;
constexpr uint32_t kMagic = 0x31425755u;  // "UWB1"
constexpr uint32_t kFormatVersion = 1;
constexpr int64_t kMaxElems = (int64_t(1) << 31) - 256;

// Decode-table entry (derived from the code lengths):
//   bits  0..4   bits consumed by the decoded symbols (1..12)
//   bits  5..9   4 x number of symbols decoded from the 12-bit window (4..20)
//   bit  10      the window starts with no valid code (only in incomplete
//                codes): decoded as one symbol 0 of 12 bits, and reported
//   bits 11..30  up to five symbols, symbol i in bits 11+4i..14+4i
constexpr int kLutMaxSymbols = 5;
constexpr int kLutSymShift = 11;
__host__ __device__ constexpr uint32_t lut_bits(uint32_t e) { return e & 31u; }
__host__ __device__ constexpr uint32_t lut_nibble_bits(uint32_t e) { return (e >> 5) & 31u; }
constexpr uint32_t kLutInvalid = 1u << 10;

struct Geometry {
    int64_t N = 0, K = 0, n = 0, G = 0, GW = 0, KG = 0, NW = 0, nseg = 0, nchunk = 0;
    static Geometry of(int64_t N, int64_t K);
};

}  // namespace uw

struct uw_blob {
    uint32_t magic = uw::kMagic;
    uw::Geometry geo;
    uint32_t forms = 0;
    int64_t V = 0;
    uint8_t palette[16] = {0};
    uint8_t inv[256] = {0};
    uint8_t code_len[16] = {0};
    uint32_t code[16] = {0};
    uint64_t freq[16] = {0};
    uint64_t hist[256] = {0};
    uint64_t total_bits = 0;
    int64_t nwords = 0;
    uint64_t off[UW_NSECT] = {0};
    uint64_t bytes[UW_NSECT] = {0};
    uint64_t dev_bytes = 0;
    uint8_t* dev = nullptr;      // committed device image (caller-owned)
    bool committed = false;
    // compress-time host state (between query and commit)
    std::vector<uint32_t> vbits_h, vpre_h;
    std::vector<uint64_t> chunk_off_h;
    std::vector<uint16_t> seg_rel_h;
    std::vector<uint32_t> lut_h;

    const uint8_t* sec(int s) const { return dev + off[s]; }
};

namespace uw {

// ---- host helpers (uw_host.cpp)
void build_code(const uint64_t freq[16], uint8_t len[16], uint32_t code[16]);
void build_lut(const uint8_t len[16], const uint32_t code[16], uint32_t* lut);
void layout_sections(uw_blob* b);
int num_sms();

// ---- device status words (one per kernel translation unit)
int decode_status_take();
int gemm_status_take();

// ---- compress kernels (uw_compress.cu)
struct CompressScratch {
    uint32_t* hist;     // [256]
    uint32_t* freq;     // [16]
    uint32_t* vbits;    // [GW]
    uint32_t* segbits;  // [nseg]
};
size_t compress_scratch_bytes(const Geometry& g);
CompressScratch carve_scratch(void* base, const Geometry& g);
cudaError_t launch_histogram(const uint16_t* W, int64_t n, uint32_t* hist, cudaStream_t s);
cudaError_t launch_verbatim_freq(const uint16_t* W, const Geometry& g, const uint8_t inv[256],
                                 uint32_t* vbits, uint32_t* freq, cudaStream_t s);
cudaError_t launch_segbits(const uint16_t* W, const Geometry& g, const uint8_t inv[256],
                           const uint32_t* vbits, const uint8_t len[16], uint32_t* segbits,
                           cudaStream_t s);
cudaError_t launch_planes(const uint16_t* W, const Geometry& g, const uint8_t inv[256],
                          const uint32_t* vbits, uint8_t* sm, uint8_t* idx, cudaStream_t s);
cudaError_t launch_vexp(const uint16_t* W, const Geometry& g, const uint32_t* vbits,
                        const uint32_t* vpre, uint8_t* vexp, cudaStream_t s);
cudaError_t launch_vcol(const Geometry& g, const uint32_t* vbits, uint32_t* vcol, cudaStream_t s);
cudaError_t launch_encode(const uint16_t* W, const Geometry& g, const uint8_t inv[256],
                          const uint32_t* vbits, const uint8_t len[16], const uint32_t code[16],
                          const uint64_t* chunk_off, const uint16_t* seg_rel, uint32_t* stream,
                          int64_t nwords, cudaStream_t s);

// ---- decoders (uw_decode.cu)
enum DecodeMode { kDecodeFull = 0, kDecodeExponent = 1, kDecodeTranscode = 2 };
// Standalone decoder; `sms` > 0 stands in for the device's SM count.
cudaError_t launch_decode(const uw_blob* b, int mode, void* out, int sms, cudaStream_t s);
// Decoder that runs beside the GEMM: `ctas` CTAs of 4 warps, each finished
// 8192-weight task counted in band_ready[task / (K/64)] under call tag `epoch`.
cudaError_t launch_decode_beside(const uw_blob* b, int mode, void* out, int ctas, unsigned long long* band_ready,
                                 unsigned long long epoch, cudaStream_t s);
constexpr int kDecodeBesideSmem = (1 << 12) * 4 + 4 * 32 * 32 * 4;   // LUT + 4 warps of staging
// Standalone decoder launch shape for `ntasks` warp tasks: CTAs and warps a
// CTA (one CTA per SM, every warp the same number of tasks at most).
void decode_grid(int64_t ntasks, int sms, int* grid, int* warps);
// Fused Huffman-decode GEMV/small-batch product (no decoded plane in HBM):
// Y[M,N] = X[M,K] . W^T straight from the Huffman form, M <= kFusedMaxM per
// launch, K a multiple of 256.  Workspace: fused_ws_bytes.
constexpr int kFusedMaxM = 16;
size_t fused_ws_bytes(int64_t M, int64_t N, int64_t K);
cudaError_t launch_fused_huffman(const uw_blob* b, const uint16_t* X, int64_t M, void* Y, int out_f32, void* ws,
                                 size_t ws_bytes, cudaStream_t s, uw_status* st);

// ---- GEMM (uw_gemm.cu)
enum GemmSource { kSrcDense = 0, kSrcExponent = 1, kSrcPalette = 2 };
struct GemmArgs {
    int src = kSrcDense;
    const uint16_t* X = nullptr;
    int64_t M = 0, N = 0, K = 0;
    const uint16_t* W = nullptr;      // dense source
    const uint8_t* sm = nullptr;      // sign+mantissa plane
    const uint8_t* ex = nullptr;      // exponent plane (exponent source)
    const uint8_t* idx = nullptr;     // index plane (palette source)
    const uint32_t* vbits = nullptr;
    const uint32_t* vpre = nullptr;
    const uint8_t* vexp = nullptr;
    const uint32_t* vcol = nullptr;
    const uint8_t* palette = nullptr; // host array of 16
    void* Y = nullptr;
    int out_f32 = 0;
    int variant = UW_VARIANT_AUTO;
    int grid = 0;
    int split_k = 0;                  // >0: k ranges per output tile (grid ignored)
    int stages = 0;                   // >0: cap on the stage ring depth
    void* ws = nullptr;               // partial sums + tile counters
    size_t ws_bytes = 0;
    int smem_cap = 0;                 // >0: dynamic shared memory limit (room for a decoder CTA)
    unsigned long long epoch = 0;     // 0: a fresh call tag
    const unsigned long long* band_ready = nullptr;   // decoder-beside-GEMM readiness
    int64_t band_tasks = 0, ntasks = 0;
    int static_sm = 0;                // sm plane and verbatim flags read from the committed blob (no kernel writes it)
    int static_s2 = 0;                // second plane too (the stored index plane)
    // paired call (gate and up, direct palette, SwiGLU epilogue): the up
    // projection's planes; Y = silu(X.Wg^T) * (X.Wu^T)
    int pair = 0;
    // SwiGLU in three launches: the launch writes its accumulators per tile
    // (float4 columns of 128 rows, m_tiles * n_tiles * MG * 128 floats) to
    // gate_out instead of Y; launch_swiglu_blocks then combines two of them
    float* gate_out = nullptr;
    const uint8_t* sm2 = nullptr;
    const uint8_t* idx2 = nullptr;
    const uint32_t* vbits2 = nullptr;
    const uint32_t* vpre2 = nullptr;
    const uint8_t* vexp2 = nullptr;
    const uint32_t* vcol2 = nullptr;
    const uint8_t* palette2 = nullptr;
};
// Work split of the tensor-core kernel: batch tile MG, stage k KB, tiles,
// (tile, k step) iterations and CTA count P.  fixup: some tile is cut
// between CTAs (partial sums and tags in the workspace).  ok = false when the
// options are inconsistent (split_k >= 2 with more CTAs than SMs).
struct GemmSplit {
    int MG = 16, KB = 64, m_tiles = 0, n_tiles = 0, kt = 0, P = 0;
    int64_t tiles = 0, total = 0;
    bool fixup = false, ok = true;
};
GemmSplit gemm_split(int64_t M, int64_t N, int64_t K, int grid, int split_k, int nh = 1);
size_t gemm_ws_bytes(int64_t M, int64_t N, int64_t K, int grid, int split_k, int nh = 1);
// Tensor-core GEMM; the calls gemv_serves() accepts (by the variant, or with
// UW_VARIANT_AUTO batch 1 on a projection with few 128-row tiles and no
// decoder beside) go to the CUDA-core GEMV instead.
cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s, uw_status* st);
// H = silu(G) * U from two tile-block arrays written with gate_out (same
// M, N, K, grid and split_k as the launches that wrote them)
cudaError_t launch_swiglu_blocks(const float* G, const float* U, void* H, int64_t M, int64_t N, int64_t K, int grid,
                                 int split_k, int out_f32, cudaStream_t s);
bool gemv_serves(const GemmArgs& a);
constexpr int kGemvMaxM = 1;   // batches the GEMV kernel supports
cudaError_t launch_gemv(const GemmArgs& a, cudaStream_t s, uw_status* st);
int gemm_default_grid();
unsigned long long gemm_next_epoch();

}  // namespace uw
