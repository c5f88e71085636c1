// uw_host.cpp -- host side of libunweight: argument checks, the Huffman code
// construction, the device-image layout, compress/serialize/deserialize, and
// the dispatch of the four pipelines and of the autotuner.
//
// "Cloudflare推出Unweight無損壓縮系統" (easyvibecoding.app):
//   §BF16權重壓縮原理  palette of the 16 most frequent exponents, Huffman code,
//                      verbatim 64-weight rows;
//   §四種執行管道      pipelines (full / exponent / transcode / direct palette);
//   §自動調優機制      coordinate-descent autotuner measured on the hardware.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "uw_internal.h"

namespace uw {

Geometry Geometry::of(int64_t N, int64_t K) {
    Geometry g;
    g.N = N;
    g.K = K;
    g.n = N * K;
    g.G = g.n / kGroup;
    g.GW = (g.G + 31) / 32;
    g.KG = K / kGroup;
    g.NW = 4 * ((N + 127) / 128);
    g.nseg = (g.n + kSeg - 1) / kSeg;
    g.nchunk = (g.nseg + kChunkSegs - 1) / kChunkSegs;
    return g;
}

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = v > 0 ? v : 148;
    }
    return cached[dev];
}

// ---------------------------------------------------------------------------
// Optimal length-limited code lengths (package-merge), kept as per-level lists
// of tags.  The deepest level holds the leaves -- used symbols ordered by
// (count, symbol).  Each shallower level merges the leaves with the pairs
// ("packages") of the level below; on equal weight a leaf goes first.  Then,
// from the top level down: the first 2(n-1) items are taken; every leaf taken
// at some level lengthens its symbol's code by one, and the k packages taken
// at one level mean the first 2k items of the level below are taken.
// ---------------------------------------------------------------------------
void build_code(const uint64_t freq[16], uint8_t len[16], uint32_t code[16]) {
    for (int s = 0; s < 16; s++) { len[s] = 0; code[s] = 0; }
    std::vector<int> used;
    for (int s = 0; s < 16; s++)
        if (freq[s]) used.push_back(s);
    std::stable_sort(used.begin(), used.end(), [&](int a, int b) { return freq[a] < freq[b]; });
    const int n = (int)used.size();
    if (n == 1) len[used[0]] = 1;
    if (n >= 2) {
        struct Tag { uint64_t w; int leaf; };   // leaf < 0: package
        std::vector<std::vector<Tag>> level(kLmax + 1);
        for (int i = 0; i < n; i++) level[kLmax].push_back({freq[used[i]], i});
        for (int l = kLmax - 1; l >= 1; l--) {
            const std::vector<Tag>& below = level[l + 1];
            std::vector<uint64_t> pk;
            for (size_t i = 0; i + 1 < below.size(); i += 2) pk.push_back(below[i].w + below[i + 1].w);
            size_t a = 0, b = 0;
            while (a < (size_t)n || b < pk.size()) {
                bool leaf = b >= pk.size() || (a < (size_t)n && freq[used[a]] <= pk[b]);
                if (leaf) { level[l].push_back({freq[used[a]], (int)a}); a++; }
                else { level[l].push_back({pk[b], -1}); b++; }
            }
        }
        size_t take = 2 * (size_t)(n - 1);
        for (int l = 1; l <= kLmax && take; l++) {
            size_t packages = 0;
            for (size_t i = 0; i < take && i < level[l].size(); i++) {
                if (level[l][i].leaf >= 0) len[used[level[l][i].leaf]]++;
                else packages++;
            }
            take = 2 * packages;
        }
    }
    // canonical assignment: by (length, symbol); a longer code continues the
    // running count shifted left by the length difference
    std::vector<int> order;
    for (int s = 0; s < 16; s++)
        if (len[s]) order.push_back(s);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return len[a] < len[b]; });
    uint32_t c = 0;
    int prev = order.empty() ? 0 : len[order[0]];
    for (size_t i = 0; i < order.size(); i++) {
        int s = order[i];
        c <<= (len[s] - prev);
        prev = len[s];
        code[s] = c++;
    }
}

// 4096-entry multi-symbol table: entry p decodes as many whole codes (up to
// five) as fit in the 12-bit window p, read MSB first.
void build_lut(const uint8_t len[16], const uint32_t code[16], uint32_t* lut) {
    std::vector<int> one_sym(kLutSize, -1), one_len(kLutSize, 0);
    for (int s = 0; s < 16; s++) {
        if (!len[s]) continue;
        uint32_t lo = code[s] << (kLmax - len[s]), hi = (code[s] + 1) << (kLmax - len[s]);
        for (uint32_t p = lo; p < hi && p < (uint32_t)kLutSize; p++) { one_sym[p] = s; one_len[p] = len[s]; }
    }
    for (uint32_t p = 0; p < (uint32_t)kLutSize; p++) {
        uint32_t syms = 0, nsym = 0, used = 0;
        while (nsym < (uint32_t)kLutMaxSymbols) {
            uint32_t w = (p << used) & (kLutSize - 1);
            if (one_sym[w] < 0 || used + one_len[w] > (uint32_t)kLmax) break;
            syms |= (uint32_t)one_sym[w] << (4 * nsym);
            used += one_len[w];
            nsym++;
        }
        if (nsym == 0)   // no valid code: progress by 12 bits, flag it
            lut[p] = 12u | (4u << 5) | kLutInvalid;
        else
            lut[p] = used | ((4 * nsym) << 5) | (syms << kLutSymShift);
    }
}

static uint64_t al256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

void layout_sections(uw_blob* b) {
    const Geometry& g = b->geo;
    const bool huff = b->forms & UW_FORM_HUFFMAN, pal = b->forms & UW_FORM_PALETTE;
    b->bytes[UW_SEC_SM] = g.n;
    b->bytes[UW_SEC_VBITS] = g.GW * 4;
    b->bytes[UW_SEC_VPRE] = g.GW * 4;
    b->bytes[UW_SEC_VEXP] = b->V * kGroup;
    b->bytes[UW_SEC_VCOL] = g.KG * g.NW * 4;
    b->bytes[UW_SEC_IDX] = pal ? g.n / 2 : 0;
    b->bytes[UW_SEC_STREAM] = huff ? b->nwords * 4 : 0;
    b->bytes[UW_SEC_CHUNK_OFF] = huff ? g.nchunk * 8 : 0;
    b->bytes[UW_SEC_SEG_REL] = huff ? g.nseg * 2 : 0;
    b->bytes[UW_SEC_LUT] = huff ? kLutSize * 4 : 0;
    uint64_t off = 0;
    for (int s = 0; s < UW_NSECT; s++) {
        b->off[s] = off;
        off += al256(b->bytes[s]);
    }
    b->dev_bytes = off < 256 ? 256 : off;
}

static void palette_from_hist(const uint64_t hist[256], uint8_t palette[16], uint8_t inv[256]) {
    std::vector<int> e(256);
    for (int i = 0; i < 256; i++) e[i] = i;
    std::stable_sort(e.begin(), e.end(), [&](int a, int b) { return hist[a] > hist[b]; });
    memset(inv, 0xFF, 256);
    for (int i = 0; i < 16; i++) {
        palette[i] = (uint8_t)e[i];
        inv[e[i]] = (uint8_t)i;
    }
}

}  // namespace uw

using namespace uw;

// ===========================================================================
// misc
// ===========================================================================
extern "C" const char* uw_status_str(int s) {
    switch (s) {
        case UW_OK: return "UW_OK";
        case UW_ERR_INVALID_ARG: return "UW_ERR_INVALID_ARG";
        case UW_ERR_SHAPE: return "UW_ERR_SHAPE";
        case UW_ERR_CORRUPT: return "UW_ERR_CORRUPT";
        case UW_ERR_UNSUPPORTED: return "UW_ERR_UNSUPPORTED";
        case UW_ERR_WORKSPACE: return "UW_ERR_WORKSPACE";
        case UW_ERR_CUDA: return "UW_ERR_CUDA";
        case UW_ERR_TIMEOUT: return "UW_ERR_TIMEOUT";
        case UW_ERR_DEVICE: return "UW_ERR_DEVICE";
        default: return "UW_ERR_UNKNOWN";
    }
}

extern "C" int uw_version(void) { return 10100; }

extern "C" uw_status uw_last_device_status(void* stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) {
        cudaGetLastError();
        return UW_ERR_CUDA;
    }
    int d = decode_status_take(), g = gemm_status_take();
    if (d < 0 || g < 0) return UW_ERR_CUDA;
    return (uw_status)(d ? d : g);
}

static bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

static uw_status check_shape(int64_t N, int64_t K) {
    if (N < 1 || K < kGroup || K % kGroup) return UW_ERR_SHAPE;
    if (N > kMaxElems / K) return UW_ERR_SHAPE;
    return UW_OK;
}

static uw_status cuda_ok(cudaError_t e) {
    if (e == cudaSuccess) return UW_OK;
    cudaGetLastError();
    return UW_ERR_CUDA;
}

// ===========================================================================
// compress
// ===========================================================================
extern "C" uw_status uw_compress_scratch_bytes(int64_t N, int64_t K, size_t* bytes) {
    if (!bytes) return UW_ERR_INVALID_ARG;
    uw_status st = check_shape(N, K);
    if (st) return st;
    *bytes = compress_scratch_bytes(Geometry::of(N, K));
    return UW_OK;
}

extern "C" uw_status uw_compress_query(const uint16_t* W, int64_t N, int64_t K, uint32_t forms, void* scratch,
                                       size_t scratch_bytes, void* stream, uw_blob** out, size_t* dev_bytes) {
    if (!W || !scratch || !out || !dev_bytes) return UW_ERR_INVALID_ARG;
    if (forms == 0 || (forms & ~uint32_t(UW_FORM_HUFFMAN | UW_FORM_PALETTE))) return UW_ERR_INVALID_ARG;
    uw_status st = check_shape(N, K);
    if (st) return st;
    if (!aligned(W, 16) || !aligned(scratch, 256)) return UW_ERR_INVALID_ARG;
    Geometry g = Geometry::of(N, K);
    if (scratch_bytes < compress_scratch_bytes(g)) return UW_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    CompressScratch sc = carve_scratch(scratch, g);

    uw_blob* b = new uw_blob();
    b->geo = g;
    b->forms = forms;
    auto fail = [&](uw_status e) { delete b; return e; };

    std::vector<uint32_t> h32(256), f32(16);
    if (cuda_ok(launch_histogram(W, g.n, sc.hist, s))) return fail(UW_ERR_CUDA);
    if (cuda_ok(cudaMemcpyAsync(h32.data(), sc.hist, 256 * 4, cudaMemcpyDeviceToHost, s))) return fail(UW_ERR_CUDA);
    if (cuda_ok(cudaStreamSynchronize(s))) return fail(UW_ERR_CUDA);
    for (int i = 0; i < 256; i++) b->hist[i] = h32[i];
    palette_from_hist(b->hist, b->palette, b->inv);

    if (cuda_ok(launch_verbatim_freq(W, g, b->inv, sc.vbits, sc.freq, s))) return fail(UW_ERR_CUDA);
    b->vbits_h.resize(g.GW);
    if (cuda_ok(cudaMemcpyAsync(f32.data(), sc.freq, 16 * 4, cudaMemcpyDeviceToHost, s))) return fail(UW_ERR_CUDA);
    if (cuda_ok(cudaMemcpyAsync(b->vbits_h.data(), sc.vbits, g.GW * 4, cudaMemcpyDeviceToHost, s)))
        return fail(UW_ERR_CUDA);
    if (cuda_ok(cudaStreamSynchronize(s))) return fail(UW_ERR_CUDA);
    for (int i = 0; i < 16; i++) b->freq[i] = f32[i];
    build_code(b->freq, b->code_len, b->code);

    b->vpre_h.resize(g.GW);
    uint64_t run = 0;
    for (int64_t w = 0; w < g.GW; w++) {
        b->vpre_h[w] = (uint32_t)run;
        run += __builtin_popcount(b->vbits_h[w]);
    }
    b->V = (int64_t)run;

    if (forms & UW_FORM_HUFFMAN) {
        std::vector<uint32_t> segbits(g.nseg);
        if (cuda_ok(launch_segbits(W, g, b->inv, sc.vbits, b->code_len, sc.segbits, s))) return fail(UW_ERR_CUDA);
        if (cuda_ok(cudaMemcpyAsync(segbits.data(), sc.segbits, g.nseg * 4, cudaMemcpyDeviceToHost, s)))
            return fail(UW_ERR_CUDA);
        if (cuda_ok(cudaStreamSynchronize(s))) return fail(UW_ERR_CUDA);
        b->chunk_off_h.resize(g.nchunk);
        b->seg_rel_h.resize(g.nseg);
        uint64_t pos = 0;
        for (int64_t j = 0; j < g.nseg; j++) {
            if (j % kChunkSegs == 0) b->chunk_off_h[j / kChunkSegs] = pos;
            b->seg_rel_h[j] = (uint16_t)(pos - b->chunk_off_h[j / kChunkSegs]);
            pos += segbits[j];
        }
        b->total_bits = pos;
        b->nwords = (int64_t)((pos + 31) / 32) + 2;
        b->lut_h.resize(kLutSize);
        build_lut(b->code_len, b->code, b->lut_h.data());
    }
    layout_sections(b);
    *out = b;
    *dev_bytes = b->dev_bytes;
    return UW_OK;
}

extern "C" uw_status uw_compress_commit(uw_blob* b, const uint16_t* W, void* scratch, size_t scratch_bytes,
                                        void* dev_buf, size_t dev_bytes, void* stream) {
    if (!b || b->magic != kMagic || !W || !scratch || !dev_buf) return UW_ERR_INVALID_ARG;
    if (b->committed) return UW_ERR_INVALID_ARG;
    const Geometry& g = b->geo;
    if (scratch_bytes < compress_scratch_bytes(g)) return UW_ERR_WORKSPACE;
    if (!aligned(dev_buf, 256) || dev_bytes < b->dev_bytes) return UW_ERR_WORKSPACE;
    if (!aligned(W, 16)) return UW_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    b->dev = (uint8_t*)dev_buf;
    uint8_t* d = b->dev;
    auto sec = [&](int k) { return d + b->off[k]; };
    if (cuda_ok(cudaMemsetAsync(d, 0, b->dev_bytes, s))) return UW_ERR_CUDA;
    if (cuda_ok(cudaMemcpyAsync(sec(UW_SEC_VBITS), b->vbits_h.data(), g.GW * 4, cudaMemcpyHostToDevice, s)))
        return UW_ERR_CUDA;
    if (cuda_ok(cudaMemcpyAsync(sec(UW_SEC_VPRE), b->vpre_h.data(), g.GW * 4, cudaMemcpyHostToDevice, s)))
        return UW_ERR_CUDA;
    const uint32_t* vbits = (const uint32_t*)sec(UW_SEC_VBITS);
    if (cuda_ok(launch_planes(W, g, b->inv, vbits, sec(UW_SEC_SM),
                              (b->forms & UW_FORM_PALETTE) ? sec(UW_SEC_IDX) : nullptr, s)))
        return UW_ERR_CUDA;
    if (b->V && cuda_ok(launch_vexp(W, g, vbits, (const uint32_t*)sec(UW_SEC_VPRE), sec(UW_SEC_VEXP), s)))
        return UW_ERR_CUDA;
    if (cuda_ok(launch_vcol(g, vbits, (uint32_t*)sec(UW_SEC_VCOL), s))) return UW_ERR_CUDA;
    if (b->forms & UW_FORM_HUFFMAN) {
        if (cuda_ok(cudaMemcpyAsync(sec(UW_SEC_CHUNK_OFF), b->chunk_off_h.data(), g.nchunk * 8,
                                    cudaMemcpyHostToDevice, s)))
            return UW_ERR_CUDA;
        if (cuda_ok(cudaMemcpyAsync(sec(UW_SEC_SEG_REL), b->seg_rel_h.data(), g.nseg * 2, cudaMemcpyHostToDevice, s)))
            return UW_ERR_CUDA;
        if (cuda_ok(cudaMemcpyAsync(sec(UW_SEC_LUT), b->lut_h.data(), kLutSize * 4, cudaMemcpyHostToDevice, s)))
            return UW_ERR_CUDA;
        if (cuda_ok(launch_encode(W, g, b->inv, vbits, b->code_len, b->code, (const uint64_t*)sec(UW_SEC_CHUNK_OFF),
                                  (const uint16_t*)sec(UW_SEC_SEG_REL), (uint32_t*)sec(UW_SEC_STREAM), b->nwords, s)))
            return UW_ERR_CUDA;
    }
    if (cuda_ok(cudaStreamSynchronize(s))) return UW_ERR_CUDA;
    b->committed = true;
    std::vector<uint32_t>().swap(b->vbits_h);
    std::vector<uint32_t>().swap(b->vpre_h);
    std::vector<uint64_t>().swap(b->chunk_off_h);
    std::vector<uint16_t>().swap(b->seg_rel_h);
    std::vector<uint32_t>().swap(b->lut_h);
    return UW_OK;
}

extern "C" void uw_blob_free(uw_blob* b) {
    if (b && b->magic == kMagic) {
        b->magic = 0;
        delete b;
    }
}

extern "C" uw_status uw_blob_info_get(const uw_blob* b, uw_blob_info* info) {
    if (!b || b->magic != kMagic || !info) return UW_ERR_INVALID_ARG;
    memset(info, 0, sizeof(*info));
    const Geometry& g = b->geo;
    info->N = g.N;
    info->K = g.K;
    info->G = g.G;
    info->V = b->V;
    info->nseg = g.nseg;
    info->nchunk = g.nchunk;
    info->forms = b->forms;
    memcpy(info->palette, b->palette, 16);
    memcpy(info->code_len, b->code_len, 16);
    for (int i = 0; i < 16; i++) info->freq[i] = b->freq[i];
    for (int i = 0; i < 256; i++) info->hist[i] = b->hist[i];
    info->total_bits = b->total_bits;
    const uint64_t vstore = g.GW * 8 + b->V * kGroup;
    info->bytes_huffman_form = g.n + b->nwords * 4 + g.nchunk * 8 + g.nseg * 2 + vstore;
    info->bytes_palette_form = g.n + g.n / 2 + vstore + g.KG * g.NW * 4;
    info->device_bytes = b->dev_bytes;
    info->mean_code_len = g.n ? (double)b->total_bits / (double)g.n : 0.0;
    double H = 0.0, cover = 0.0;
    for (int e = 0; e < 256; e++) {
        if (!b->hist[e]) continue;
        double p = (double)b->hist[e] / (double)g.n;
        H -= p * std::log2(p);
    }
    for (int i = 0; i < 16; i++) cover += (double)b->hist[b->palette[i]];
    info->exponent_entropy = H;
    info->palette_coverage = cover / (double)g.n;
    for (int s = 0; s < UW_NSECT; s++) {
        info->section_offset[s] = b->off[s];
        info->section_bytes[s] = b->bytes[s];
    }
    return UW_OK;
}

extern "C" uw_status uw_blob_section(const uw_blob* b, int section, const void** dev_ptr, size_t* bytes) {
    if (!b || b->magic != kMagic || !dev_ptr || !bytes || section < 0 || section >= UW_NSECT) return UW_ERR_INVALID_ARG;
    if (!b->committed) return UW_ERR_INVALID_ARG;
    *dev_ptr = b->dev + b->off[section];
    *bytes = b->bytes[section];
    return UW_OK;
}

// ===========================================================================
// serialize / deserialize ("distribution bundle")
// ===========================================================================
namespace {
struct SerialHeader {
    uint32_t magic, version;
    int64_t N, K;
    uint32_t forms, pad;
    int64_t V, nwords;
    uint64_t total_bits;
    uint8_t palette[16], code_len[16];
    uint64_t freq[16], hist[256];
    uint64_t bytes[UW_NSECT];
};
constexpr int kSerialSections = UW_SEC_LUT;   // LUT is derived, not stored
}  // namespace

extern "C" uw_status uw_blob_serialized_bytes(const uw_blob* b, size_t* bytes) {
    if (!b || b->magic != kMagic || !bytes || !b->committed) return UW_ERR_INVALID_ARG;
    size_t t = sizeof(SerialHeader);
    for (int s = 0; s < kSerialSections; s++) t += b->bytes[s];
    *bytes = t;
    return UW_OK;
}

extern "C" uw_status uw_blob_serialize(const uw_blob* b, void* host_dst, size_t cap, size_t* written, void* stream) {
    size_t need = 0;
    uw_status st = uw_blob_serialized_bytes(b, &need);
    if (st) return st;
    if (!host_dst || cap < need) return UW_ERR_WORKSPACE;
    SerialHeader h{};
    h.magic = kMagic;
    h.version = kFormatVersion;
    h.N = b->geo.N;
    h.K = b->geo.K;
    h.forms = b->forms;
    h.V = b->V;
    h.nwords = b->nwords;
    h.total_bits = b->total_bits;
    memcpy(h.palette, b->palette, 16);
    memcpy(h.code_len, b->code_len, 16);
    for (int i = 0; i < 16; i++) h.freq[i] = b->freq[i];
    for (int i = 0; i < 256; i++) h.hist[i] = b->hist[i];
    for (int s = 0; s < UW_NSECT; s++) h.bytes[s] = s < kSerialSections ? b->bytes[s] : 0;
    uint8_t* p = (uint8_t*)host_dst;
    memcpy(p, &h, sizeof h);
    p += sizeof h;
    cudaStream_t s = (cudaStream_t)stream;
    for (int k = 0; k < kSerialSections; k++) {
        if (b->bytes[k] && cuda_ok(cudaMemcpyAsync(p, b->dev + b->off[k], b->bytes[k], cudaMemcpyDeviceToHost, s)))
            return UW_ERR_CUDA;
        p += b->bytes[k];
    }
    if (cuda_ok(cudaStreamSynchronize(s))) return UW_ERR_CUDA;
    if (written) *written = need;
    return UW_OK;
}

// Builds a handle from a header, checking everything that can be checked
// without the sections.  Returns null on inconsistency.
static uw_blob* blob_from_header(const void* host_src, size_t n) {
    if (!host_src || n < sizeof(SerialHeader)) return nullptr;
    SerialHeader h;
    memcpy(&h, host_src, sizeof h);
    if (h.magic != kMagic || h.version != kFormatVersion) return nullptr;
    if (check_shape(h.N, h.K) != UW_OK) return nullptr;
    if (h.forms == 0 || (h.forms & ~uint32_t(UW_FORM_HUFFMAN | UW_FORM_PALETTE))) return nullptr;
    Geometry g = Geometry::of(h.N, h.K);
    if (h.V < 0 || h.V > g.G) return nullptr;
    uw_blob* b = new uw_blob();
    b->geo = g;
    b->forms = h.forms;
    b->V = h.V;
    b->nwords = h.nwords;
    b->total_bits = h.total_bits;
    memcpy(b->palette, h.palette, 16);
    memcpy(b->code_len, h.code_len, 16);
    for (int i = 0; i < 16; i++) b->freq[i] = h.freq[i];
    for (int i = 0; i < 256; i++) b->hist[i] = h.hist[i];
    bool ok = true;
    // palette: distinct values
    bool seen[256] = {false};
    memset(b->inv, 0xFF, 256);
    for (int i = 0; i < 16; i++) {
        if (seen[b->palette[i]]) ok = false;
        seen[b->palette[i]] = true;
        b->inv[b->palette[i]] = (uint8_t)i;
    }
    uint64_t hsum = 0, fsum = 0;
    for (int i = 0; i < 256; i++) hsum += b->hist[i];
    for (int i = 0; i < 16; i++) fsum += b->freq[i];
    if (hsum != (uint64_t)g.n || fsum != (uint64_t)g.n) ok = false;
    if (b->forms & UW_FORM_HUFFMAN) {
        // code lengths: <= 12, used exactly by the symbols that occur, prefix-free (Kraft <= 1)
        uint64_t kraft = 0;
        int used = 0;
        for (int i = 0; i < 16; i++) {
            if (b->code_len[i] > kLmax) ok = false;
            if ((b->code_len[i] != 0) != (b->freq[i] != 0)) ok = false;
            if (b->code_len[i]) { kraft += 1ull << (kLmax - b->code_len[i]); used++; }
        }
        if (kraft > (1ull << kLmax) || used == 0) ok = false;
        if (used >= 2 && kraft != (1ull << kLmax)) ok = false;
        uint64_t bits = 0;
        for (int i = 0; i < 16; i++) bits += b->freq[i] * b->code_len[i];
        if (bits != b->total_bits) ok = false;
        if (b->nwords != (int64_t)((b->total_bits + 31) / 32) + 2) ok = false;
        if (ok) {
            // canonical codes follow from the stored lengths alone
            std::vector<int> order;
            for (int s = 0; s < 16; s++)
                if (b->code_len[s]) order.push_back(s);
            std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return b->code_len[x] < b->code_len[y]; });
            uint32_t c = 0;
            int prev = order.empty() ? 0 : b->code_len[order[0]];
            for (int s : order) {
                c <<= (b->code_len[s] - prev);
                prev = b->code_len[s];
                b->code[s] = c++;
            }
        }
    } else {
        b->nwords = 0;
        b->total_bits = 0;
    }
    if (!ok) { delete b; return nullptr; }
    layout_sections(b);
    for (int s = 0; s < kSerialSections; s++)
        if (h.bytes[s] != b->bytes[s]) { delete b; return nullptr; }
    size_t need = sizeof h;
    for (int s = 0; s < kSerialSections; s++) need += b->bytes[s];
    if (n < need) { delete b; return nullptr; }
    return b;
}

extern "C" uw_status uw_blob_device_bytes(const void* host_src, size_t n, size_t* dev_bytes) {
    if (!dev_bytes) return UW_ERR_INVALID_ARG;
    uw_blob* b = blob_from_header(host_src, n);
    if (!b) return UW_ERR_CORRUPT;
    *dev_bytes = b->dev_bytes;
    delete b;
    return UW_OK;
}

extern "C" uw_status uw_blob_deserialize(const void* host_src, size_t n, void* dev_buf, size_t dev_bytes, void* stream,
                                         uw_blob** out) {
    if (!out || !dev_buf) return UW_ERR_INVALID_ARG;
    uw_blob* b = blob_from_header(host_src, n);
    if (!b) return UW_ERR_CORRUPT;
    if (!aligned(dev_buf, 256) || dev_bytes < b->dev_bytes) { delete b; return UW_ERR_WORKSPACE; }
    const Geometry& g = b->geo;
    const uint8_t* p = (const uint8_t*)host_src + sizeof(SerialHeader);
    const uint8_t* sec[UW_NSECT] = {nullptr};
    for (int s = 0; s < kSerialSections; s++) { sec[s] = p; p += b->bytes[s]; }
    // verbatim store consistency
    const uint32_t* vbits = (const uint32_t*)sec[UW_SEC_VBITS];
    const uint32_t* vpre = (const uint32_t*)sec[UW_SEC_VPRE];
    uint64_t run = 0;
    bool ok = true;
    for (int64_t w = 0; w < g.GW; w++) {
        if (vpre[w] != run) ok = false;
        run += __builtin_popcount(vbits[w]);
    }
    if (g.G & 31) {
        uint32_t tail = vbits[g.GW - 1] >> (g.G & 31);
        if (tail) ok = false;
    }
    if (run != (uint64_t)b->V) ok = false;
    // vcol must be the transpose of vbits
    {
        const uint32_t* vcol = (const uint32_t*)sec[UW_SEC_VCOL];
        uint64_t colbits = 0;
        for (int64_t t = 0; t < g.KG * g.NW; t++) colbits += __builtin_popcount(vcol[t]);
        if (colbits != run) ok = false;
        for (int64_t gi = 0; ok && gi < g.G; gi++) {
            if (!((vbits[gi >> 5] >> (gi & 31)) & 1u)) continue;
            int64_t nn = gi / g.KG, kt = gi % g.KG;
            if (!((vcol[kt * g.NW + nn / 32] >> (nn % 32)) & 1u)) ok = false;
        }
    }
    if (b->forms & UW_FORM_HUFFMAN) {
        const uint64_t* co = (const uint64_t*)sec[UW_SEC_CHUNK_OFF];
        const uint16_t* sr = (const uint16_t*)sec[UW_SEC_SEG_REL];
        if (g.nchunk && co[0] != 0) ok = false;
        for (int64_t c = 0; ok && c < g.nchunk; c++) {
            if (c && co[c] < co[c - 1]) ok = false;
            if (co[c] > b->total_bits) ok = false;
        }
        for (int64_t j = 0; ok && j < g.nseg; j++) {
            uint64_t pos = co[j / kChunkSegs] + sr[j];
            if (j % kChunkSegs == 0 && sr[j] != 0) ok = false;
            if (pos > b->total_bits) ok = false;
            if ((uint64_t)sr[j] > (uint64_t)(j % kChunkSegs) * kSeg * kLmax) ok = false;
        }
    }
    if (!ok) { delete b; return UW_ERR_CORRUPT; }
    cudaStream_t s = (cudaStream_t)stream;
    b->dev = (uint8_t*)dev_buf;
    for (int k = 0; k < kSerialSections; k++)
        if (b->bytes[k] && cuda_ok(cudaMemcpyAsync(b->dev + b->off[k], sec[k], b->bytes[k], cudaMemcpyHostToDevice, s))) {
            delete b;
            return UW_ERR_CUDA;
        }
    if (b->forms & UW_FORM_HUFFMAN) {
        b->lut_h.resize(kLutSize);
        build_lut(b->code_len, b->code, b->lut_h.data());
        if (cuda_ok(cudaMemcpyAsync(b->dev + b->off[UW_SEC_LUT], b->lut_h.data(), kLutSize * 4, cudaMemcpyHostToDevice, s))) {
            delete b;
            return UW_ERR_CUDA;
        }
    }
    if (cuda_ok(cudaStreamSynchronize(s))) { delete b; return UW_ERR_CUDA; }
    std::vector<uint32_t>().swap(b->lut_h);
    b->committed = true;
    *out = b;
    return UW_OK;
}

// ===========================================================================
// decode
// ===========================================================================
static uw_status check_committed(const uw_blob* b) {
    if (!b || b->magic != kMagic || !b->committed) return UW_ERR_INVALID_ARG;
    return UW_OK;
}

static uw_status decode_common(const uw_blob* b, void* out, int mode, void* stream) {
    uw_status st = check_committed(b);
    if (st) return st;
    if (!out || !aligned(out, 16)) return UW_ERR_INVALID_ARG;
    if (!(b->forms & UW_FORM_HUFFMAN)) return UW_ERR_UNSUPPORTED;
    return cuda_ok(launch_decode(b, mode, out, 0, (cudaStream_t)stream));
}

extern "C" uw_status uw_decode_full(const uw_blob* b, uint16_t* W_out, void* stream) {
    return decode_common(b, W_out, kDecodeFull, stream);
}
extern "C" uw_status uw_decode_exponent(const uw_blob* b, uint8_t* E_out, void* stream) {
    return decode_common(b, E_out, kDecodeExponent, stream);
}
extern "C" uw_status uw_transcode_palette(const uw_blob* b, uint8_t* idx_out, void* stream) {
    return decode_common(b, idx_out, kDecodeTranscode, stream);
}

// ===========================================================================
// GEMM
// ===========================================================================
static size_t decode_buffer_bytes(const uw_blob* b, int pipeline) {
    switch (pipeline) {
        case UW_PIPE_FULL: return al256(b->geo.n * 2);
        case UW_PIPE_EXPONENT: return al256(b->geo.n);
        case UW_PIPE_TRANSCODE: return al256(b->geo.n / 2);
        default: return 0;
    }
}

static bool runs_beside(const uw_gemm_opts* o) {
    return o->sm_dec > 0 && o->pipeline != UW_PIPE_DIRECT_PALETTE && o->pipeline != UW_PIPE_FUSED_HUFFMAN;
}

static size_t band_counter_bytes(const uw_blob* b) { return al256((uint64_t)((b->geo.N + 127) / 128) * 8); }

extern "C" uw_status uw_plan_resolve(const uw_gemm_opts* o, int64_t M, uw_gemm_opts* out) {
    if (!o || !out || M < 0) return UW_ERR_INVALID_ARG;
    *out = *o;
    if (o->pipeline != UW_PIPE_AUTO) return UW_OK;
    if (!o->plan || o->plan_entries <= 0) return UW_ERR_INVALID_ARG;
    // exact M, else the largest tuned M below it, else the smallest tuned M
    const uw_plan_entry* exact = nullptr, *below = nullptr, *lowest = nullptr;
    for (int i = 0; i < o->plan_entries; i++) {
        const uw_plan_entry& e = o->plan[i];
        if (e.blob_index != o->projection) continue;
        if (e.M == M && !exact) exact = &e;
        if (e.M <= M && (!below || e.M > below->M)) below = &e;
        if (!lowest || e.M < lowest->M) lowest = &e;
    }
    const uw_plan_entry* e = exact ? exact : below ? below : lowest;
    if (!e || e->pipeline < UW_PIPE_FULL || e->pipeline > UW_PIPE_FUSED_HUFFMAN) return UW_ERR_INVALID_ARG;
    out->pipeline = e->pipeline;
    out->variant = e->variant;
    out->sm_dec = e->sm_dec;
    out->grid = e->grid;
    out->split_k = e->split_k;
    out->plan = nullptr;
    out->plan_entries = 0;
    return UW_OK;
}

static uw_status check_opts(const uw_gemm_opts* o) {
    if (o->pipeline < UW_PIPE_FULL || o->pipeline > UW_PIPE_FUSED_HUFFMAN) return UW_ERR_INVALID_ARG;
    if (o->sm_dec < 0 || o->grid < 0 || o->split_k < 0 || o->stages < 0) return UW_ERR_INVALID_ARG;
    if (o->variant < UW_VARIANT_AUTO || o->variant > UW_VARIANT_GEMV) return UW_ERR_INVALID_ARG;
    return UW_OK;
}

extern "C" uw_status uw_gemm_workspace(const uw_blob* b, int64_t M, const uw_gemm_opts* oin, size_t* bytes) {
    uw_status st = check_committed(b);
    if (st) return st;
    if (!oin || !bytes || M < 0) return UW_ERR_INVALID_ARG;
    uw_gemm_opts ov;
    st = uw_plan_resolve(oin, M, &ov);
    if (st) return st;
    const uw_gemm_opts* o = &ov;
    st = check_opts(o);
    if (st) return st;
    if (M == 0) { *bytes = 0; return UW_OK; }
    if (o->pipeline == UW_PIPE_FUSED_HUFFMAN) {
        *bytes = al256(fused_ws_bytes(M, b->geo.N, b->geo.K));
        return UW_OK;
    }
    *bytes = decode_buffer_bytes(b, o->pipeline) + al256(gemm_ws_bytes(M, b->geo.N, b->geo.K, o->grid, o->split_k)) +
             (runs_beside(o) ? band_counter_bytes(b) : 0);
    return UW_OK;
}

// Side stream and fork/join events per device for the decoder-beside-GEMM
// launch (§解壓與運算資源共享).  Created once; calls on one device that run
// beside each other must not overlap (they share these).
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    cudaEvent_t done[2] = {nullptr, nullptr};    // layer sequences: decode buffer b filled
    cudaEvent_t freed[2] = {nullptr, nullptr};   // layer sequences: decode buffer b read by its GEMM
};
static SideStream* side_stream(uw_status* st) {
    static std::mutex mu;
    static SideStream per_dev[64];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        *st = UW_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    SideStream& ss = per_dev[dev];
    if (!ss.s) {
        bool ok = cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) == cudaSuccess &&
                  cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) == cudaSuccess;
        for (int b = 0; b < 2 && ok; b++)
            ok = cudaEventCreateWithFlags(&ss.done[b], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&ss.freed[b], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            cudaGetLastError();
            *st = UW_ERR_CUDA;
            return nullptr;
        }
    }
    return &ss;
}

// Test hook (UW_DEBUG_SKIP_DECODER=1): a decoder-beside-GEMM call launches
// only its GEMM, whose bounded waits for decoded bands then run out.
static bool debug_skip_decoder() {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("UW_DEBUG_SKIP_DECODER");
        v = (e && e[0] == '1') ? 1 : 0;
    }
    return v == 1;
}

extern "C" uw_status uw_gemm(const uint16_t* X, int64_t M, const uw_blob* b, void* Y, const uw_gemm_opts* oin,
                             void* stream) {
    uw_status st = check_committed(b);
    if (st) return st;
    if (!oin || M < 0) return UW_ERR_INVALID_ARG;
    uw_gemm_opts ov;
    st = uw_plan_resolve(oin, M, &ov);
    if (st) return st;
    const uw_gemm_opts* o = &ov;
    st = check_opts(o);
    if (st) return st;
    if (M == 0) return UW_OK;
    if (!X || !Y || !aligned(X, 16) || !aligned(Y, 16)) return UW_ERR_INVALID_ARG;
    const bool needs_huff = o->pipeline != UW_PIPE_DIRECT_PALETTE;
    if (needs_huff && !(b->forms & UW_FORM_HUFFMAN)) return UW_ERR_UNSUPPORTED;
    if (!needs_huff && !(b->forms & UW_FORM_PALETTE)) return UW_ERR_UNSUPPORTED;
    if (runs_beside(o) && o->variant == UW_VARIANT_GEMV) return UW_ERR_UNSUPPORTED;
    size_t need = 0;
    uw_gemm_workspace(b, M, o, &need);
    if (!o->workspace || o->workspace_bytes < need || !aligned(o->workspace, 256)) return UW_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* ws = (uint8_t*)o->workspace;
    if (o->pipeline == UW_PIPE_FUSED_HUFFMAN) {
        // one pass per kFusedMaxM batch rows; each pass decodes the stream again
        if (b->geo.K % kSeg) return UW_ERR_UNSUPPORTED;
        const size_t ysz = o->out_f32 ? 4 : 2;
        for (int64_t m0 = 0; m0 < M; m0 += kFusedMaxM) {
            const int64_t mc = M - m0 < kFusedMaxM ? M - m0 : kFusedMaxM;
            cudaError_t e = launch_fused_huffman(b, X + m0 * b->geo.K, mc, (uint8_t*)Y + (size_t)m0 * b->geo.N * ysz,
                                                 o->out_f32 ? 1 : 0, ws, o->workspace_bytes, s, &st);
            if (st) return st;
            if (cuda_ok(e)) return UW_ERR_CUDA;
        }
        return UW_OK;
    }
    const size_t dbuf = decode_buffer_bytes(b, o->pipeline);

    GemmArgs a;
    a.X = X;
    a.M = M;
    a.N = b->geo.N;
    a.K = b->geo.K;
    a.Y = Y;
    a.out_f32 = o->out_f32 ? 1 : 0;
    a.variant = o->variant;
    a.grid = o->grid;
    a.split_k = o->split_k;
    a.stages = o->stages;
    a.ws = ws + dbuf;
    a.ws_bytes = o->workspace_bytes - dbuf;
    a.sm = b->sec(UW_SEC_SM);
    a.vbits = (const uint32_t*)b->sec(UW_SEC_VBITS);
    a.vpre = (const uint32_t*)b->sec(UW_SEC_VPRE);
    a.vexp = b->sec(UW_SEC_VEXP);
    a.vcol = (const uint32_t*)b->sec(UW_SEC_VCOL);
    a.palette = b->palette;
    a.static_sm = 1;   // the sign+mantissa plane and verbatim flags are the committed blob's
    const int mode = o->pipeline == UW_PIPE_FULL ? kDecodeFull : o->pipeline == UW_PIPE_EXPONENT ? kDecodeExponent
                                                                                                : kDecodeTranscode;
    switch (o->pipeline) {
        case UW_PIPE_FULL: a.src = kSrcDense; a.W = (const uint16_t*)ws; break;
        case UW_PIPE_EXPONENT: a.src = kSrcExponent; a.ex = ws; break;
        case UW_PIPE_TRANSCODE: a.src = kSrcPalette; a.idx = ws; break;
        default:   // the committed blob's index plane: no kernel writes it
            a.src = kSrcPalette;
            a.idx = b->sec(UW_SEC_IDX);
            a.static_s2 = 1;
            break;
    }
    if (o->pipeline == UW_PIPE_DIRECT_PALETTE) {
        cudaError_t e = launch_gemm(a, s, &st);
        if (st) return st;
        return cuda_ok(e);
    }
    if (!runs_beside(o)) {
        // decode, then GEMM
        if (cuda_ok(launch_decode(b, mode, ws, 0, s))) return UW_ERR_CUDA;
        cudaError_t e = launch_gemm(a, s, &st);
        if (st) return st;
        return cuda_ok(e);
    }
    // decoder beside the GEMM: the decoder's CTAs publish finished 128-row
    // bands, the GEMM's producer waits for a band before loading its tiles.
    // The GEMM keeps room for one decoder CTA on every SM.
    SideStream* ss = side_stream(&st);
    if (!ss) return st;
    a.ws_bytes = al256(gemm_ws_bytes(M, b->geo.N, b->geo.K, o->grid, o->split_k));
    unsigned long long* band = (unsigned long long*)(ws + dbuf + a.ws_bytes);
    a.epoch = gemm_next_epoch();
    a.band_ready = band;
    a.band_tasks = b->geo.KG;
    a.ntasks = (b->geo.n + 8191) / 8192;
    a.smem_cap = 228 * 1024 - kDecodeBesideSmem - 2048;
    if (cuda_ok(cudaEventRecord(ss->fork, s)) || cuda_ok(cudaStreamWaitEvent(ss->s, ss->fork, 0))) return UW_ERR_CUDA;
    if (!debug_skip_decoder() && cuda_ok(launch_decode_beside(b, mode, ws, o->sm_dec, band, a.epoch, s)))
        return UW_ERR_CUDA;
    cudaError_t e = launch_gemm(a, ss->s, &st);
    if (!st && e == cudaSuccess) e = cudaEventRecord(ss->join, ss->s);
    if (!st && e == cudaSuccess) e = cudaStreamWaitEvent(s, ss->join, 0);
    if (st) return st;
    return cuda_ok(e);
}

// ===========================================================================
// layer sequences with "hard" and "easy" projections (§跨層管道化)
// ===========================================================================
// Workspace: two index-plane buffers (the largest hard item's plane each)
// then the GEMM scratch (the largest item's), shared by the items in turn.
static void sequence_layout(const uw_seq_item* items, int n, int64_t M, size_t* plane, size_t* gemm) {
    *plane = 0;
    *gemm = 0;
    for (int i = 0; i < n; i++) {
        const uw_blob* b = items[i].blob;
        if (items[i].hard) *plane = std::max(*plane, (size_t)al256(b->geo.n / 2));
        *gemm = std::max(*gemm, (size_t)al256(gemm_ws_bytes(M, b->geo.N, b->geo.K, 0, 0)));
    }
}

static uw_status sequence_check(const uw_seq_item* items, int n, int64_t M, bool need_ptrs) {
    if (!items || n < 1 || M < 0) return UW_ERR_INVALID_ARG;
    for (int i = 0; i < n; i++) {
        uw_status st = check_committed(items[i].blob);
        if (st) return st;
        const unsigned need = items[i].hard ? UW_FORM_HUFFMAN : UW_FORM_PALETTE;
        if (!(items[i].blob->forms & need)) return UW_ERR_UNSUPPORTED;
        if (need_ptrs && M > 0 &&
            (!items[i].X || !items[i].Y || !aligned(items[i].X, 16) || !aligned(items[i].Y, 16)))
            return UW_ERR_INVALID_ARG;
    }
    return UW_OK;
}

extern "C" uw_status uw_sequence_workspace(const uw_seq_item* items, int n, int64_t M, size_t* bytes) {
    if (!bytes) return UW_ERR_INVALID_ARG;
    uw_status st = sequence_check(items, n, M, false);
    if (st) return st;
    size_t plane = 0, gemm = 0;
    sequence_layout(items, n, M, &plane, &gemm);
    *bytes = M ? 2 * plane + gemm : 0;
    return UW_OK;
}

extern "C" uw_status uw_gemm_sequence(const uw_seq_item* items, int n, int64_t M, int out_f32, int dec_ctas,
                                      void* workspace, size_t workspace_bytes, void* stream) {
    uw_status st = sequence_check(items, n, M, true);
    if (st) return st;
    if (dec_ctas < 0) return UW_ERR_INVALID_ARG;
    if (M == 0) return UW_OK;
    size_t plane = 0, gemm = 0;
    sequence_layout(items, n, M, &plane, &gemm);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < 2 * plane + gemm) return UW_ERR_WORKSPACE;
    uint8_t* ws = (uint8_t*)workspace;
    uint8_t* buf[2] = {ws, ws + plane};
    uint8_t* gws = ws + 2 * plane;
    cudaStream_t s = (cudaStream_t)stream;
    bool any_hard = false;
    for (int i = 0; i < n; i++) any_hard = any_hard || items[i].hard;
    SideStream* ss = nullptr;
    if (any_hard) {
        ss = side_stream(&st);
        if (!ss) return st;
        // decodes write this call's buffers: after the work already on `stream`
        if (cuda_ok(cudaEventRecord(ss->fork, s)) || cuda_ok(cudaStreamWaitEvent(ss->s, ss->fork, 0)))
            return UW_ERR_CUDA;
    }
    // with decoder CTAs beside the GEMMs, every GEMM leaves room for one
    const int smem_cap = dec_ctas > 0 ? 228 * 1024 - kDecodeBesideSmem - 2048 : 0;
    int h = 0;                 // hard items so far
    for (int i = 0; i < n; i++) {
        const uw_seq_item& it = items[i];
        const uw_blob* b = it.blob;
        GemmArgs a;
        a.src = kSrcPalette;
        a.X = it.X;
        a.M = M;
        a.N = b->geo.N;
        a.K = b->geo.K;
        a.Y = it.Y;
        a.out_f32 = out_f32 ? 1 : 0;
        a.variant = UW_VARIANT_TENSOR;
        a.ws = gws;
        a.ws_bytes = gemm;
        a.sm = b->sec(UW_SEC_SM);
        a.vbits = (const uint32_t*)b->sec(UW_SEC_VBITS);
        a.vpre = (const uint32_t*)b->sec(UW_SEC_VPRE);
        a.vexp = b->sec(UW_SEC_VEXP);
        a.vcol = (const uint32_t*)b->sec(UW_SEC_VCOL);
        a.palette = b->palette;
        a.static_sm = 1;
        a.smem_cap = smem_cap;
        if (it.hard) {
            // the transcode of this item runs on the side stream as soon as its
            // buffer's previous GEMM (two hard items back) has read it, i.e.
            // ahead of the GEMMs in between
            const int bi = h & 1;
            if (h >= 2 && cuda_ok(cudaStreamWaitEvent(ss->s, ss->freed[bi], 0))) return UW_ERR_CUDA;
            cudaError_t e = dec_ctas > 0 ? launch_decode_beside(b, kDecodeTranscode, buf[bi], dec_ctas, nullptr, 0, ss->s)
                                         : launch_decode(b, kDecodeTranscode, buf[bi], 0, ss->s);
            if (cuda_ok(e) || cuda_ok(cudaEventRecord(ss->done[bi], ss->s)) ||
                cuda_ok(cudaStreamWaitEvent(s, ss->done[bi], 0)))
                return UW_ERR_CUDA;
            a.idx = buf[bi];
            a.static_s2 = 0;
            cudaError_t eg = launch_gemm(a, s, &st);
            if (st) return st;
            if (cuda_ok(eg) || cuda_ok(cudaEventRecord(ss->freed[bi], s))) return UW_ERR_CUDA;
            h++;
        } else {
            a.idx = b->sec(UW_SEC_IDX);
            a.static_s2 = 1;
            cudaError_t eg = launch_gemm(a, s, &st);
            if (st) return st;
            if (cuda_ok(eg)) return UW_ERR_CUDA;
        }
    }
    if (any_hard) {
        // the side stream joins back (its last decode is already awaited by a GEMM)
        if (cuda_ok(cudaEventRecord(ss->join, ss->s)) || cuda_ok(cudaStreamWaitEvent(s, ss->join, 0)))
            return UW_ERR_CUDA;
    }
    return UW_OK;
}

// ===========================================================================
// gate + up with the SwiGLU epilogue (§未來方向)
// ===========================================================================
static uw_status swiglu_check(const uw_blob* g, const uw_blob* u, int64_t M, const uw_gemm_opts* o) {
    uw_status st = check_committed(g);
    if (st) return st;
    st = check_committed(u);
    if (st) return st;
    if (!o || M < 0) return UW_ERR_INVALID_ARG;
    st = check_opts(o);
    if (st) return st;
    if (g->geo.N != u->geo.N || g->geo.K != u->geo.K) return UW_ERR_SHAPE;
    if (o->pipeline != UW_PIPE_DIRECT_PALETTE || o->variant == UW_VARIANT_GEMV || o->sm_dec != 0)
        return UW_ERR_UNSUPPORTED;
    if (!(g->forms & UW_FORM_PALETTE) || !(u->forms & UW_FORM_PALETTE)) return UW_ERR_UNSUPPORTED;
    return UW_OK;
}

// Batches above 128 rows run the SwiGLU in three launches: a paired tile
// (gate and up accumulators side by side in TMEM) is capped at 128 batch
// rows, which doubles the rebuild work per product against the
// single-matrix kernel's 256-row tiles.  The gate and the up launch write
// their fp32 products into the workspace per tile; a third, elementwise
// kernel writes H = silu(G) * U.  (Reading G in the up launch's epilogue was
// slower: one epilogue warp per sub-partition waits on the loads chunk by
// chunk.)
static bool swiglu_split(int64_t M) { return M > 128; }
static size_t swiglu_gate_bytes(const uw_blob* g, int64_t M, const uw_gemm_opts* o) {
    const GemmSplit sp = gemm_split(M, g->geo.N, g->geo.K, o->grid, o->split_k, 1);
    return al256((size_t)sp.tiles * (size_t)sp.MG * 128 * 4);
}
static size_t swiglu_ws_bytes(const uw_blob* g, int64_t M, const uw_gemm_opts* o) {
    if (!swiglu_split(M)) return al256(gemm_ws_bytes(M, g->geo.N, g->geo.K, o->grid, o->split_k, 2));
    return 2 * swiglu_gate_bytes(g, M, o) + al256(gemm_ws_bytes(M, g->geo.N, g->geo.K, o->grid, o->split_k, 1));
}

static void set_palette_planes(GemmArgs& a, const uw_blob* b) {
    a.sm = b->sec(UW_SEC_SM);
    a.idx = b->sec(UW_SEC_IDX);
    a.vbits = (const uint32_t*)b->sec(UW_SEC_VBITS);
    a.vpre = (const uint32_t*)b->sec(UW_SEC_VPRE);
    a.vexp = b->sec(UW_SEC_VEXP);
    a.vcol = (const uint32_t*)b->sec(UW_SEC_VCOL);
    a.palette = b->palette;
}

extern "C" uw_status uw_gemm_swiglu_workspace(const uw_blob* g, const uw_blob* u, int64_t M, const uw_gemm_opts* o,
                                              size_t* bytes) {
    if (!bytes) return UW_ERR_INVALID_ARG;
    uw_status st = swiglu_check(g, u, M, o);
    if (st) return st;
    *bytes = M ? swiglu_ws_bytes(g, M, o) : 0;
    return UW_OK;
}

extern "C" uw_status uw_gemm_swiglu(const uint16_t* X, int64_t M, const uw_blob* g, const uw_blob* u, void* H,
                                    const uw_gemm_opts* o, void* stream) {
    uw_status st = swiglu_check(g, u, M, o);
    if (st) return st;
    if (M == 0) return UW_OK;
    if (!X || !H || !aligned(X, 16) || !aligned(H, 16)) return UW_ERR_INVALID_ARG;
    const size_t need = swiglu_ws_bytes(g, M, o);
    if (!o->workspace || o->workspace_bytes < need || !aligned(o->workspace, 256)) return UW_ERR_WORKSPACE;
    if (swiglu_split(M)) {
        const size_t gbytes = swiglu_gate_bytes(g, M, o);
        float* G = (float*)o->workspace;
        float* U = (float*)((uint8_t*)o->workspace + gbytes);
        GemmArgs a;
        a.src = kSrcPalette;
        a.X = X;
        a.M = M;
        a.N = g->geo.N;
        a.K = g->geo.K;
        a.variant = o->variant;
        a.grid = o->grid;
        a.split_k = o->split_k;
        a.stages = o->stages;
        a.ws = (uint8_t*)o->workspace + 2 * gbytes;
        a.ws_bytes = o->workspace_bytes - 2 * gbytes;
        a.static_sm = 1;
        a.static_s2 = 1;
        set_palette_planes(a, g);
        a.Y = H;                // not written: the accumulators go to G, then U
        a.out_f32 = o->out_f32 ? 1 : 0;
        a.gate_out = G;
        cudaError_t e = launch_gemm(a, (cudaStream_t)stream, &st);
        if (st) return st;
        if (cuda_ok(e)) return UW_ERR_CUDA;
        set_palette_planes(a, u);
        a.gate_out = U;
        e = launch_gemm(a, (cudaStream_t)stream, &st);
        if (st) return st;
        if (cuda_ok(e)) return UW_ERR_CUDA;
        return cuda_ok(launch_swiglu_blocks(G, U, H, M, g->geo.N, g->geo.K, o->grid, o->split_k, o->out_f32 ? 1 : 0,
                                            (cudaStream_t)stream));
    }
    GemmArgs a;
    a.src = kSrcPalette;
    a.pair = 1;
    a.X = X;
    a.M = M;
    a.N = g->geo.N;
    a.K = g->geo.K;
    a.Y = H;
    a.out_f32 = o->out_f32 ? 1 : 0;
    a.variant = o->variant;
    a.grid = o->grid;
    a.split_k = o->split_k;
    a.stages = o->stages;
    a.ws = o->workspace;
    a.ws_bytes = o->workspace_bytes;
    a.static_sm = 1;
    a.static_s2 = 1;
    a.sm = g->sec(UW_SEC_SM);
    a.idx = g->sec(UW_SEC_IDX);
    a.vbits = (const uint32_t*)g->sec(UW_SEC_VBITS);
    a.vpre = (const uint32_t*)g->sec(UW_SEC_VPRE);
    a.vexp = g->sec(UW_SEC_VEXP);
    a.vcol = (const uint32_t*)g->sec(UW_SEC_VCOL);
    a.palette = g->palette;
    a.sm2 = u->sec(UW_SEC_SM);
    a.idx2 = u->sec(UW_SEC_IDX);
    a.vbits2 = (const uint32_t*)u->sec(UW_SEC_VBITS);
    a.vpre2 = (const uint32_t*)u->sec(UW_SEC_VPRE);
    a.vexp2 = u->sec(UW_SEC_VEXP);
    a.vcol2 = (const uint32_t*)u->sec(UW_SEC_VCOL);
    a.palette2 = u->palette;
    cudaError_t e = launch_gemm(a, (cudaStream_t)stream, &st);
    if (st) return st;
    return cuda_ok(e);
}

extern "C" uw_status uw_dense_gemm_workspace(int64_t M, int64_t N, int64_t K, int variant, int grid, int split_k,
                                             size_t* bytes) {
    if (!bytes || M < 0 || grid < 0 || split_k < 0) return UW_ERR_INVALID_ARG;
    if (variant < UW_VARIANT_AUTO || variant > UW_VARIANT_GEMV) return UW_ERR_INVALID_ARG;
    uw_status st = check_shape(N, K);
    if (st) return st;
    *bytes = M ? gemm_ws_bytes(M, N, K, grid, split_k) : 0;
    return UW_OK;
}

extern "C" uw_status uw_dense_gemm(const uint16_t* X, int64_t M, const uint16_t* W, int64_t N, int64_t K, void* Y,
                                   int out_f32, int variant, int grid, int split_k, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    if (M < 0 || grid < 0 || split_k < 0) return UW_ERR_INVALID_ARG;
    if (variant < UW_VARIANT_AUTO || variant > UW_VARIANT_GEMV) return UW_ERR_INVALID_ARG;
    uw_status st = check_shape(N, K);
    if (st) return st;
    if (M == 0) return UW_OK;
    if (!X || !W || !Y || !aligned(X, 16) || !aligned(W, 16) || !aligned(Y, 16)) return UW_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < gemm_ws_bytes(M, N, K, grid, split_k))
        return UW_ERR_WORKSPACE;
    GemmArgs a;
    a.src = kSrcDense;
    a.X = X;
    a.M = M;
    a.N = N;
    a.K = K;
    a.W = W;
    a.Y = Y;
    a.out_f32 = out_f32 ? 1 : 0;
    a.variant = variant;
    a.grid = grid;
    a.split_k = split_k;
    a.ws = workspace;
    a.ws_bytes = workspace_bytes;
    cudaError_t e = launch_gemm(a, (cudaStream_t)stream, &st);
    if (st) return st;
    return cuda_ok(e);
}

// ===========================================================================
// autotune (§自動調優機制)
// ===========================================================================
namespace {

const char* kPipeNames[] = {"full", "exponent", "transcode", "direct_palette", "fused_huffman"};

struct Cand {
    int pipe, variant, grid, split_k, sm_dec;
    bool operator==(const Cand& o) const {
        return pipe == o.pipe && variant == o.variant && grid == o.grid && split_k == o.split_k && sm_dec == o.sm_dec;
    }
};

uw_gemm_opts cand_opts(const Cand& c, void* ws, size_t wsb) {
    uw_gemm_opts o{};
    o.pipeline = c.pipe;
    o.variant = c.variant;
    o.grid = c.grid;
    o.split_k = c.split_k;
    o.sm_dec = c.sm_dec;
    o.workspace = ws;
    o.workspace_bytes = wsb;
    return o;
}

// The kernel path and work split a candidate leads to, so that candidates
// that run the same thing are measured once.
struct PathKey {
    int pipe, gemv, P, sm_dec;
    bool operator==(const PathKey& o) const { return pipe == o.pipe && gemv == o.gemv && P == o.P && sm_dec == o.sm_dec; }
};

PathKey path_of(const Cand& c, const uw_blob* b, int64_t M) {
    if (c.pipe == UW_PIPE_FUSED_HUFFMAN) return PathKey{c.pipe, 0, 0, 0};
    GemmArgs a;
    a.M = M;
    a.N = b->geo.N;
    a.K = b->geo.K;
    a.variant = c.variant;
    a.grid = c.grid;
    a.split_k = c.split_k;
    const bool beside = c.sm_dec > 0 && c.pipe != UW_PIPE_DIRECT_PALETTE;
    const bool gemv = !beside && gemv_serves(a);
    PathKey k{c.pipe, gemv ? 1 : 0, gemv ? 0 : gemm_split(M, a.N, a.K, c.grid, c.split_k).P, beside ? c.sm_dec : 0};
    return k;
}

// Feasible candidates of one projection at batch M, one per distinct path.
std::vector<Cand> candidates(const uw_blob* b, int64_t M, size_t wsb) {
    const int sms = num_sms();
    std::vector<Cand> raw;
    for (int pp = UW_PIPE_FULL; pp <= UW_PIPE_DIRECT_PALETTE; pp++) {
        raw.push_back({pp, UW_VARIANT_AUTO, 0, 0, 0});
        if (M == 1) {
            raw.push_back({pp, UW_VARIANT_TENSOR, 0, 0, 0});
            raw.push_back({pp, UW_VARIANT_GEMV, 0, 0, 0});
        }
        raw.push_back({pp, UW_VARIANT_TENSOR, sms, 0, 0});       // stream-K over one CTA per SM
        raw.push_back({pp, UW_VARIANT_TENSOR, 0, 1, 0});         // one CTA per output tile
        if (pp != UW_PIPE_DIRECT_PALETTE)
            for (int f : {1, 2, 4}) raw.push_back({pp, UW_VARIANT_AUTO, 0, 0, f * sms / 2});
    }
    if (M <= kFusedMaxM && b->geo.K % kSeg == 0) raw.push_back({UW_PIPE_FUSED_HUFFMAN, UW_VARIANT_AUTO, 0, 0, 0});
    std::vector<Cand> out;
    std::vector<PathKey> seen;
    for (const Cand& c : raw) {
        const bool has = c.pipe == UW_PIPE_DIRECT_PALETTE ? (b->forms & UW_FORM_PALETTE) : (b->forms & UW_FORM_HUFFMAN);
        if (!has) continue;
        if (c.split_k > 0 && !gemm_split(M, b->geo.N, b->geo.K, c.grid, c.split_k).ok) continue;
        uw_gemm_opts o = cand_opts(c, nullptr, 0);
        size_t need = 0;
        if (uw_gemm_workspace(b, M, &o, &need) != UW_OK || need > wsb) continue;
        const PathKey k = path_of(c, b, M);
        bool dup = false;
        for (const PathKey& s : seen) dup = dup || s == k;
        if (dup) continue;
        seen.push_back(k);
        out.push_back(c);
    }
    return out;
}

struct Trial {
    int64_t M;
    int round, proj;
    Cand c;
    double layer_us;
};

}  // namespace

extern "C" uw_status uw_autotune(const uw_blob* const* blobs, int nproj, int ncopies, const int64_t* Ms, int nM,
                                 const uint16_t* const* X, void* const* Y, void* workspace, size_t workspace_bytes,
                                 int reps, uw_plan_entry* plan, const char* plan_json_path, void* stream) {
    if (!blobs || nproj < 1 || ncopies < 1 || !Ms || nM < 1 || !X || !Y || !plan || reps < 1) return UW_ERR_INVALID_ARG;
    for (int c = 0; c < ncopies; c++)
        for (int i = 0; i < nproj; i++) {
            const uw_blob* b = blobs[c * nproj + i];
            uw_status st = check_committed(b);
            if (st) return st;
            if (b->geo.N != blobs[i]->geo.N || b->geo.K != blobs[i]->geo.K) return UW_ERR_SHAPE;
        }
    for (int i = 0; i < nproj; i++)
        if (!X[i] || !Y[i]) return UW_ERR_INVALID_ARG;
    for (int m = 0; m < nM; m++)
        if (Ms[m] < 1) return UW_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    cudaEvent_t e0, e1;
    if (cuda_ok(cudaEventCreate(&e0))) return UW_ERR_CUDA;
    if (cuda_ok(cudaEventCreate(&e1))) { cudaEventDestroy(e0); return UW_ERR_CUDA; }
    // a call refused, a launch that failed, or a device status raised (a
    // bounded wait that expired) makes the candidate infeasible
    auto run_calls = [&](int64_t M, const std::vector<Cand>& ch, int only, int passes, int first_pass) -> bool {
        bool ok = true;
        for (int r = 0; r < passes; r++) {
            const int c = (first_pass + r) % ncopies;
            for (int i = 0; i < nproj; i++) {
                if (only >= 0 && i != only) continue;
                uw_gemm_opts o = cand_opts(ch[i], workspace, workspace_bytes);
                if (uw_gemm(X[i], M, blobs[c * nproj + i], Y[i], &o, stream) != UW_OK) ok = false;
            }
        }
        return ok;
    };
    // device time per pass (microseconds), or -1 if the candidate failed
    auto measure = [&](int64_t M, const std::vector<Cand>& ch, int only) -> double {
        bool ok = run_calls(M, ch, only, ncopies, 0);   // warm-up: every copy once
        if (uw_last_device_status(stream) != UW_OK) ok = false;
        if (!ok) return -1.0;
        cudaEventRecord(e0, s);
        ok = run_calls(M, ch, only, reps, 0);
        cudaEventRecord(e1, s);
        if (cudaEventSynchronize(e1) != cudaSuccess) { cudaGetLastError(); return -1.0; }
        if (uw_last_device_status(stream) != UW_OK || !ok) return -1.0;
        float ms = 0.f;
        cudaEventElapsedTime(&ms, e0, e1);
        return 1000.0 * ms / reps;
    };
    std::vector<Trial> trials;
    uw_status result = UW_OK;
    for (int mi = 0; mi < nM && result == UW_OK; mi++) {
        const int64_t M = Ms[mi];
        std::vector<std::vector<Cand>> cands(nproj);
        for (int i = 0; i < nproj; i++) {
            cands[i] = candidates(blobs[i], M, workspace_bytes);
            if (cands[i].empty()) result = UW_ERR_WORKSPACE;
        }
        if (result) break;
        // start: the first candidate that runs (pipeline 1 first, as listed)
        std::vector<Cand> choice(nproj);
        for (int i = 0; i < nproj; i++) choice[i] = cands[i][0];
        double best = measure(M, choice, -1);
        for (int i = 0; i < nproj && best < 0; i++) {
            // the first candidates failed: take, per projection, the first that runs alone
            for (const Cand& c : cands[i]) {
                std::vector<Cand> t = choice;
                t[i] = c;
                if (measure(M, t, i) >= 0) { choice[i] = c; break; }
            }
            best = measure(M, choice, -1);
        }
        if (best < 0) { result = UW_ERR_DEVICE; break; }
        for (int i = 0; i < nproj; i++) trials.push_back({M, 0, i, choice[i], best});
        for (int round = 0; round < 8; round++) {
            bool improved = false;
            for (int i = 0; i < nproj; i++) {
                for (const Cand& c : cands[i]) {
                    if (c == choice[i]) continue;
                    std::vector<Cand> trial = choice;
                    trial[i] = c;
                    const double t = measure(M, trial, -1);
                    trials.push_back({M, round, i, c, t});
                    if (t >= 0 && t < best * 0.99) { best = t; choice = trial; improved = true; }
                }
            }
            if (!improved) break;
        }
        for (int i = 0; i < nproj; i++) {
            uw_plan_entry& pe = plan[mi * nproj + i];
            pe.blob_index = i;
            pe.M = M;
            pe.pipeline = choice[i].pipe;
            pe.variant = choice[i].variant;
            pe.sm_dec = choice[i].sm_dec;
            pe.grid = choice[i].grid;
            pe.split_k = choice[i].split_k;
            pe.us = measure(M, choice, i);
            pe.layer_us = best;
        }
    }
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    if (result == UW_OK && plan_json_path) {
        FILE* f = fopen(plan_json_path, "w");
        if (!f) return UW_ERR_INVALID_ARG;
        fprintf(f, "{\"plan\": [\n");
        for (int k = 0; k < nM * nproj; k++)
            fprintf(f,
                    "  {\"projection\": %d, \"M\": %lld, \"pipeline\": \"%s\", \"variant\": %d, \"sm_dec\": %d, "
                    "\"grid\": %d, \"split_k\": %d, \"us\": %.3f, \"layer_us\": %.3f}%s\n",
                    plan[k].blob_index, (long long)plan[k].M, kPipeNames[plan[k].pipeline], plan[k].variant,
                    plan[k].sm_dec, plan[k].grid, plan[k].split_k, plan[k].us, plan[k].layer_us,
                    k + 1 < nM * nproj ? "," : "");
        fprintf(f, "],\n\"trials\": [\n");
        for (size_t k = 0; k < trials.size(); k++) {
            const Trial& t = trials[k];
            fprintf(f,
                    "  {\"M\": %lld, \"round\": %d, \"projection\": %d, \"pipeline\": \"%s\", \"variant\": %d, "
                    "\"sm_dec\": %d, \"grid\": %d, \"split_k\": %d, \"layer_us\": %.3f}%s\n",
                    (long long)t.M, t.round, t.proj, kPipeNames[t.c.pipe], t.c.variant, t.c.sm_dec, t.c.grid,
                    t.c.split_k, t.layer_us, k + 1 < trials.size() ? "," : "");
        }
        fprintf(f, "]}\n");
        fclose(f);
    }
    return result;
}

// ---------------------------------------------------------------------------
// Reads back the "plan" array written above: objects of "key": value pairs
// (numbers, or the pipeline's name as a string).
// ---------------------------------------------------------------------------
static bool json_field(const std::string& obj, const char* key, std::string* val) {
    const std::string k = std::string("\"") + key + "\"";
    size_t p = obj.find(k);
    if (p == std::string::npos) return false;
    p = obj.find(':', p + k.size());
    if (p == std::string::npos) return false;
    p++;
    while (p < obj.size() && (obj[p] == ' ' || obj[p] == '\t' || obj[p] == '\n' || obj[p] == '\r')) p++;
    if (p >= obj.size()) return false;
    if (obj[p] == '"') {
        size_t q = obj.find('"', p + 1);
        if (q == std::string::npos) return false;
        *val = obj.substr(p + 1, q - p - 1);
        return true;
    }
    size_t q = p;
    while (q < obj.size() && obj[q] != ',' && obj[q] != '}') q++;
    *val = obj.substr(p, q - p);
    return !val->empty();
}

extern "C" uw_status uw_plan_load_json(const char* path, uw_plan_entry* entries, int cap, int* n) {
    if (!path || !n || cap < 0 || (cap > 0 && !entries)) return UW_ERR_INVALID_ARG;
    FILE* f = fopen(path, "rb");
    if (!f) return UW_ERR_INVALID_ARG;
    std::string text;
    char buf[4096];
    size_t got;
    while ((got = fread(buf, 1, sizeof buf, f)) > 0) text.append(buf, got);
    fclose(f);
    size_t p = text.find("\"plan\"");
    if (p == std::string::npos) return UW_ERR_CORRUPT;
    p = text.find('[', p);
    if (p == std::string::npos) return UW_ERR_CORRUPT;
    const size_t end = text.find(']', p);
    if (end == std::string::npos) return UW_ERR_CORRUPT;
    int count = 0;
    for (;;) {
        const size_t a = text.find('{', p);
        if (a == std::string::npos || a > end) break;
        const size_t b = text.find('}', a);
        if (b == std::string::npos || b > end) return UW_ERR_CORRUPT;
        const std::string obj = text.substr(a, b - a + 1);
        uw_plan_entry e{};
        std::string v;
        if (!json_field(obj, "projection", &v)) return UW_ERR_CORRUPT;
        e.blob_index = atoi(v.c_str());
        if (!json_field(obj, "M", &v)) return UW_ERR_CORRUPT;
        e.M = atoll(v.c_str());
        if (!json_field(obj, "pipeline", &v)) return UW_ERR_CORRUPT;
        e.pipeline = -1;
        for (int k = 0; k <= UW_PIPE_FUSED_HUFFMAN; k++)
            if (v == kPipeNames[k]) e.pipeline = k;
        if (e.pipeline < 0) {
            char* q = nullptr;
            long pv = strtol(v.c_str(), &q, 10);
            if (q == v.c_str() || pv < UW_PIPE_FULL || pv > UW_PIPE_FUSED_HUFFMAN) return UW_ERR_CORRUPT;
            e.pipeline = (int32_t)pv;
        }
        if (json_field(obj, "variant", &v)) e.variant = atoi(v.c_str());
        if (json_field(obj, "sm_dec", &v)) e.sm_dec = atoi(v.c_str());
        if (json_field(obj, "grid", &v)) e.grid = atoi(v.c_str());
        if (json_field(obj, "split_k", &v)) e.split_k = atoi(v.c_str());
        if (json_field(obj, "us", &v)) e.us = atof(v.c_str());
        if (json_field(obj, "layer_us", &v)) e.layer_us = atof(v.c_str());
        if (e.M < 1 || e.blob_index < 0 || e.variant < UW_VARIANT_AUTO || e.variant > UW_VARIANT_GEMV || e.sm_dec < 0 ||
            e.grid < 0 || e.split_k < 0)
            return UW_ERR_CORRUPT;
        if (count < cap) entries[count] = e;
        count++;
        p = b + 1;
    }
    if (count == 0) return UW_ERR_CORRUPT;
    *n = count;
    return UW_OK;
}
