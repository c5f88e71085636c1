/*
 * uw_oracle.c -- plain, slow, obviously-correct CPU statement of the
 * Unweight-style lossless BF16 weight format and of Y = X . W^T.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * generator with the CUDA library; the two meet only through the seeded
 * synthetic inputs and the byte layout written down in the format spec.
 *
 * Source of the method: the web page "Cloudflare推出Unweight無損壓縮系統，將LLM
 * 模型大小壓縮15-22%" (easyvibecoding.app), sections
 *   §BF16權重壓縮原理   -- BF16 = sign(1) | exponent(8) | mantissa(7); the sign
 *                          and mantissa are kept unchanged, only the exponent
 *                          byte is entropy coded (Huffman); a handful of
 *                          exponents dominate (top 16 cover >99%, ~2.6 bits);
 *                          a 64-weight row holding an exponent outside the
 *                          16-entry palette is stored verbatim;
 *   §四種執行管道       -- full decode, exponent-only decode, palette transcode
 *                          (4-bit indices), direct palette;
 *   §重建矩陣乘法核心運作 -- the reconstructed weight feeds Y = X . W^T.
 * The pages print no bit layout, so every layout choice below is the reading
 * recorded in the design notes (group = 64 consecutive K-elements of one
 * output row; Huffman over the 16 palette indices; package-merge with a
 * 12-bit length limit; DEFLATE-style canonical codes, MSB-first; 256-symbol
 * segments with 16-segment chunks for parallel decode).
 *
 * Every function is a direct loop over the definition.  No blocking, no
 * vectorisation, no threads.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#define OR_GROUP 64          /* weights per verbatim-decision group      */
#define OR_PALETTE 16        /* palette entries                          */
#define OR_SEG 256           /* symbols per decode segment               */
#define OR_CHUNK_SEGS 16     /* segments per chunk (chunk_off entry)     */
#define OR_LMAX 12           /* longest permitted Huffman code           */

/* ---------------------------------------------------------------------- */
/* Step 1 -- split each BF16 bit pattern into its exponent byte and its   */
/* sign+mantissa byte (§BF16權重壓縮原理: 1 sign bit, 8 exponent bits,     */
/* 7 mantissa bits; sign and mantissa stay as they are).                   */
/*   bits = s eeeeeeee mmmmmmm  ->  e = eeeeeeee,  sm = s mmmmmmm          */
/* ---------------------------------------------------------------------- */
void or_split(const uint16_t *w, int64_t n, uint8_t *e, uint8_t *sm)
{
    for (int64_t i = 0; i < n; i++) {
        uint16_t b = w[i];
        uint8_t sign = (uint8_t)((b >> 15) & 1u);
        uint8_t expo = (uint8_t)((b >> 7) & 0xFFu);
        uint8_t mant = (uint8_t)(b & 0x7Fu);
        e[i] = expo;
        sm[i] = (uint8_t)((sign << 7) | mant);
    }
}

/* Inverse of or_split. */
void or_merge(const uint8_t *e, const uint8_t *sm, int64_t n, uint16_t *w)
{
    for (int64_t i = 0; i < n; i++) {
        uint16_t sign = (uint16_t)((sm[i] >> 7) & 1u);
        uint16_t mant = (uint16_t)(sm[i] & 0x7Fu);
        w[i] = (uint16_t)((sign << 15) | ((uint16_t)e[i] << 7) | mant);
    }
}

/* Step 2 -- exponent histogram over all N*K weights. */
void or_histogram(const uint8_t *e, int64_t n, uint64_t *hist /*256*/)
{
    for (int v = 0; v < 256; v++) hist[v] = 0;
    for (int64_t i = 0; i < n; i++) hist[e[i]]++;
}

/* Step 3 -- the per-matrix palette: the 16 most frequent exponents
 * (§BF16權重壓縮原理, "前16種最常見指數").  Ranking: larger count first, on
 * equal count the smaller exponent first.  Selection repeats "take the best
 * not yet taken" 16 times over all 256 values, so when fewer than 16
 * exponents occur the remaining slots are the smallest absent exponents in
 * ascending order.  inv[e] = palette position of e, or 0xFF. */
void or_palette(const uint64_t *hist, uint8_t *palette, uint8_t *inv)
{
    int taken[256];
    for (int v = 0; v < 256; v++) { taken[v] = 0; inv[v] = 0xFF; }
    for (int slot = 0; slot < OR_PALETTE; slot++) {
        int best = -1;
        for (int v = 0; v < 256; v++) {
            if (taken[v]) continue;
            if (best < 0 || hist[v] > hist[best]) best = v;
        }
        taken[best] = 1;
        palette[slot] = (uint8_t)best;
        inv[best] = (uint8_t)slot;
    }
}

/* Step 4 -- verbatim groups (§BF16權重壓縮原理, "若64權重列中任一超出前16指數
 * 調色盤，整列verbatim儲存").  Group g = 64 consecutive K-elements of row n:
 * g = n*(K/64) + k/64.  verb[g] = 1 iff some element has inv[e] == 0xFF.
 * Returns the number of verbatim groups V. */
int64_t or_verbatim(const uint8_t *e, const uint8_t *inv, int64_t N, int64_t K,
                    uint8_t *verb)
{
    int64_t groups_per_row = K / OR_GROUP, V = 0;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t kg = 0; kg < groups_per_row; kg++) {
            int64_t g = n * groups_per_row + kg;
            int out_of_palette = 0;
            for (int j = 0; j < OR_GROUP; j++) {
                int64_t i = n * K + kg * OR_GROUP + j;
                if (inv[e[i]] == 0xFF) out_of_palette = 1;
            }
            verb[g] = (uint8_t)out_of_palette;
            V += out_of_palette;
        }
    }
    return V;
}

/* Step 5 -- the symbol of every weight: its palette index, or 0 inside a
 * verbatim group (the exponent of such a weight comes from the verbatim
 * store, never from the symbol). */
void or_symbols(const uint8_t *e, const uint8_t *inv, const uint8_t *verb,
                int64_t N, int64_t K, uint8_t *s)
{
    for (int64_t i = 0; i < N * K; i++) {
        int64_t g = i / OR_GROUP;          /* row-major: i = n*K + k        */
        s[i] = verb[g] ? 0 : inv[e[i]];
    }
}

/* Step 6 -- the 4-bit index plane (§四種執行管道, "4位元調色盤索引"):
 * two symbols per byte, element 2j in the low nibble. */
void or_index_plane(const uint8_t *s, int64_t n, uint8_t *idx)
{
    for (int64_t j = 0; j < n / 2; j++)
        idx[j] = (uint8_t)((s[2 * j] & 0xF) | ((s[2 * j + 1] & 0xF) << 4));
}

/* Step 7 -- the verbatim store.
 *   vbits[w]  bit b set iff group 32w+b is verbatim (row-major group order)
 *   vpre[w]   number of verbatim groups before group 32w
 *   vexp      the 64 raw exponent bytes of each verbatim group, groups in
 *             ascending order
 *   vcol      the same flags transposed for column-tile readers: word
 *             kt*NW + n/32, bit n%32, for group (n, kt); NW = 4*ceil(N/128)
 */
void or_verbatim_store(const uint8_t *verb, const uint8_t *e, int64_t N, int64_t K,
                       uint32_t *vbits, uint32_t *vpre, uint8_t *vexp, uint32_t *vcol)
{
    int64_t G = N * K / OR_GROUP, GW = (G + 31) / 32;
    int64_t KG = K / OR_GROUP, NW = 4 * ((N + 127) / 128);
    for (int64_t w = 0; w < GW; w++) vbits[w] = 0;
    for (int64_t g = 0; g < G; g++)
        if (verb[g]) vbits[g / 32] |= (uint32_t)1u << (g % 32);
    uint32_t running = 0;
    for (int64_t w = 0; w < GW; w++) {
        vpre[w] = running;
        for (int b = 0; b < 32; b++) running += (vbits[w] >> b) & 1u;
    }
    int64_t r = 0;
    for (int64_t g = 0; g < G; g++) {
        if (!verb[g]) continue;
        for (int j = 0; j < OR_GROUP; j++) vexp[r * OR_GROUP + j] = e[g * OR_GROUP + j];
        r++;
    }
    for (int64_t t = 0; t < KG * NW; t++) vcol[t] = 0;
    for (int64_t n = 0; n < N; n++)
        for (int64_t kt = 0; kt < KG; kt++)
            if (verb[n * KG + kt]) vcol[kt * NW + n / 32] |= (uint32_t)1u << (n % 32);
}

/* Step 8 -- symbol frequencies over the whole stream. */
void or_frequencies(const uint8_t *s, int64_t n, uint64_t *freq /*16*/)
{
    for (int v = 0; v < OR_PALETTE; v++) freq[v] = 0;
    for (int64_t i = 0; i < n; i++) freq[s[i]]++;
}

/* Step 9 -- optimal length-limited Huffman code lengths by package-merge
 * (Larmore & Hirschberg 1990), code length at most lmax.
 *
 * Items are leaves (one per symbol with nonzero frequency) or packages (pairs
 * of items from the previous round).  Round 1 list = leaves sorted by
 * (frequency ascending, symbol ascending).  Each further round (lmax-1 of
 * them) pairs consecutive items of the previous list (a trailing odd item is
 * dropped) and merges those packages with the sorted leaves by weight; on
 * equal weight every leaf precedes every package, and packages keep their
 * creation order.  The first 2(n-1) items of the last list are selected and a
 * symbol's code length is the number of selected items containing its leaf.
 * One used symbol gets length 1.  Unused symbols get length 0.
 * Returns 0, or -1 when the n symbols do not fit (2^lmax < n). */
#define OR_MAXITEMS (2 * OR_PALETTE)
typedef struct { uint64_t weight; int count[OR_PALETTE]; } or_item;

int or_code_lengths(const uint64_t *freq, int lmax, uint8_t *len)
{
    int order[OR_PALETTE], n = 0;
    for (int v = 0; v < OR_PALETTE; v++) len[v] = 0;
    for (int v = 0; v < OR_PALETTE; v++) if (freq[v] > 0) order[n++] = v;
    if (n == 0) return 0;
    if (n == 1) { len[order[0]] = 1; return 0; }
    if (lmax < 31 && (1 << lmax) < n) return -1;
    /* insertion sort of the used symbols by (frequency, symbol) */
    for (int a = 1; a < n; a++) {
        int v = order[a], b = a - 1;
        while (b >= 0 && (freq[order[b]] > freq[v] ||
                          (freq[order[b]] == freq[v] && order[b] > v))) {
            order[b + 1] = order[b];
            b--;
        }
        order[b + 1] = v;
    }
    or_item leaves[OR_PALETTE];
    for (int a = 0; a < n; a++) {
        memset(&leaves[a], 0, sizeof(or_item));
        leaves[a].weight = freq[order[a]];
        leaves[a].count[order[a]] = 1;
    }
    or_item list[OR_MAXITEMS], next[OR_MAXITEMS], packages[OR_MAXITEMS];
    int list_len = n;
    for (int a = 0; a < n; a++) list[a] = leaves[a];
    for (int round = 2; round <= lmax; round++) {
        int np = list_len / 2;
        for (int p = 0; p < np; p++) {
            packages[p].weight = list[2 * p].weight + list[2 * p + 1].weight;
            for (int v = 0; v < OR_PALETTE; v++)
                packages[p].count[v] = list[2 * p].count[v] + list[2 * p + 1].count[v];
        }
        int a = 0, p = 0, m = 0;
        while (a < n || p < np) {
            int take_leaf;
            if (a >= n) take_leaf = 0;
            else if (p >= np) take_leaf = 1;
            else take_leaf = leaves[a].weight <= packages[p].weight;
            next[m++] = take_leaf ? leaves[a++] : packages[p++];
        }
        list_len = m;
        for (int t = 0; t < m; t++) list[t] = next[t];
    }
    int counts[OR_PALETTE] = {0};
    for (int t = 0; t < 2 * (n - 1); t++)
        for (int v = 0; v < OR_PALETTE; v++) counts[v] += list[t].count[v];
    for (int v = 0; v < OR_PALETTE; v++) len[v] = (uint8_t)counts[v];
    return 0;
}

/* Step 10 -- canonical code assignment as in RFC 1951 §3.2.2: count codes
 * per length, first code of each length = (first code of the previous length
 * + count of the previous length) << 1, and codes of one length go to the
 * symbols in increasing symbol order. */
void or_canonical_codes(const uint8_t *len, uint32_t *code)
{
    int bl_count[OR_LMAX + 2] = {0};
    uint32_t next_code[OR_LMAX + 2] = {0};
    for (int v = 0; v < OR_PALETTE; v++) if (len[v]) bl_count[len[v]]++;
    uint32_t c = 0;
    for (int bits = 1; bits <= OR_LMAX + 1; bits++) {
        c = (c + (uint32_t)bl_count[bits - 1]) << 1;
        next_code[bits] = c;
    }
    for (int v = 0; v < OR_PALETTE; v++) {
        code[v] = 0;
        if (len[v]) code[v] = next_code[len[v]]++;
    }
}

/* Step 11 -- stream length in bits. */
uint64_t or_stream_bits(const uint8_t *s, int64_t n, const uint8_t *len)
{
    uint64_t bits = 0;
    for (int64_t i = 0; i < n; i++) bits += len[s[i]];
    return bits;
}

/* Bit p of the stream is bit 31-(p%32) of word p/32 (MSB first). */
static void or_put_bit(uint32_t *stream, uint64_t p, uint32_t bit)
{
    if (bit) stream[p / 32] |= (uint32_t)1u << (31 - (p % 32));
}

static uint32_t or_get_bit(const uint32_t *stream, uint64_t p)
{
    return (stream[p / 32] >> (31 - (p % 32))) & 1u;
}

/* Step 12 -- encode.  Codes are written most significant bit first, back to
 * back.  The stream has nwords = ceil(bits/32) + 2 words, the tail zero.
 * chunk_off[c] = bit position of the first code of symbol 4096c;
 * seg_rel[j]   = bit position of the first code of symbol 256j minus
 *                chunk_off[j/16].                                          */
void or_encode(const uint8_t *s, int64_t n, const uint8_t *len, const uint32_t *code,
               uint32_t *stream, int64_t nwords, uint64_t *chunk_off, uint16_t *seg_rel)
{
    for (int64_t w = 0; w < nwords; w++) stream[w] = 0;
    uint64_t p = 0;
    for (int64_t i = 0; i < n; i++) {
        if (i % OR_SEG == 0) {
            int64_t j = i / OR_SEG;
            if (j % OR_CHUNK_SEGS == 0) chunk_off[j / OR_CHUNK_SEGS] = p;
            seg_rel[j] = (uint16_t)(p - chunk_off[j / OR_CHUNK_SEGS]);
        }
        for (int b = len[s[i]] - 1; b >= 0; b--) or_put_bit(stream, p++, (code[s[i]] >> b) & 1u);
    }
}

/* Step 13 -- decode `count` symbols starting at bit `p`, one bit at a time,
 * with the canonical-code rule: after reading l bits the value v is a code of
 * length l iff first[l] <= v < first[l] + n_l.  Returns the bit position
 * after the last symbol, or UINT64_MAX on an undecodable bit pattern. */
uint64_t or_decode_symbols(const uint32_t *stream, int64_t nwords, const uint8_t *len,
                           uint64_t p, int64_t count, uint8_t *out)
{
    int n_l[OR_LMAX + 1] = {0};
    uint32_t first[OR_LMAX + 1] = {0};
    uint8_t sym_by_rank[OR_PALETTE];
    int r = 0;
    for (int l = 1; l <= OR_LMAX; l++)
        for (int v = 0; v < OR_PALETTE; v++)
            if (len[v] == l) { sym_by_rank[r++] = (uint8_t)v; n_l[l]++; }
    uint32_t c = 0;
    for (int l = 1; l <= OR_LMAX; l++) { c = (c + (uint32_t)n_l[l - 1]) << 1; first[l] = c; }
    for (int64_t i = 0; i < count; i++) {
        uint32_t v = 0;
        int rank_base = 0, found = 0;
        for (int l = 1; l <= OR_LMAX; l++) {
            if (p / 32 >= (uint64_t)nwords) return UINT64_MAX;
            v = (v << 1) | or_get_bit(stream, p++);
            if (v >= first[l] && v < first[l] + (uint32_t)n_l[l]) {
                out[i] = sym_by_rank[rank_base + (int)(v - first[l])];
                found = 1;
                break;
            }
            rank_base += n_l[l];
        }
        if (!found) return UINT64_MAX;
    }
    return p;
}

/* Step 14 -- the three decoded forms (§四種執行管道).
 * Full decode: e = palette[s], or the verbatim exponent inside a verbatim
 * group; bits = sign|e|mantissa.  Exponent decode: the exponent byte alone.
 * Transcode: the index plane (identical bytes to step 6).                 */
static int64_t or_verbatim_rank(const uint32_t *vbits, const uint32_t *vpre, int64_t g)
{
    int64_t r = vpre[g / 32];
    for (int b = 0; b < (int)(g % 32); b++) r += (vbits[g / 32] >> b) & 1u;
    return r;
}

void or_exponents_from_symbols(const uint8_t *s, int64_t n, const uint8_t *palette,
                               const uint32_t *vbits, const uint32_t *vpre,
                               const uint8_t *vexp, uint8_t *e_out)
{
    for (int64_t i = 0; i < n; i++) {
        int64_t g = i / OR_GROUP;
        if ((vbits[g / 32] >> (g % 32)) & 1u)
            e_out[i] = vexp[or_verbatim_rank(vbits, vpre, g) * OR_GROUP + i % OR_GROUP];
        else
            e_out[i] = palette[s[i]];
    }
}

/* Step 15 -- the product the reconstructed weights feed
 * (§重建矩陣乘法核心運作): R[m][n] = sum_k X[m][k] * W[n][k], with X and W
 * BF16 bit patterns widened exactly.  acc_f64 = 1: double accumulation;
 * acc_f64 = 0: float accumulation in ascending k.  Products of two BF16
 * values are exact in both. */
static double or_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

void or_gemm(const uint16_t *X, const uint16_t *W, int64_t M, int64_t N, int64_t K,
             int acc_f64, double *R)
{
    for (int64_t m = 0; m < M; m++) {
        for (int64_t n = 0; n < N; n++) {
            double accd = 0.0;
            float accf = 0.0f;
            for (int64_t k = 0; k < K; k++) {
                double x = or_bf16_to_double(X[m * K + k]);
                double w = or_bf16_to_double(W[n * K + k]);
                if (acc_f64) accd += x * w;
                else accf += (float)x * (float)w;
            }
            R[m * N + n] = acc_f64 ? accd : (double)accf;
        }
    }
}

/* One output element at a time, for sampled checks at full size. */
double or_gemm_one(const uint16_t *X, const uint16_t *W, int64_t K, int64_t m, int64_t n,
                   int acc_f64)
{
    double accd = 0.0;
    float accf = 0.0f;
    for (int64_t k = 0; k < K; k++) {
        double x = or_bf16_to_double(X[m * K + k]);
        double w = or_bf16_to_double(W[n * K + k]);
        if (acc_f64) accd += x * w;
        else accf += (float)x * (float)w;
    }
    return acc_f64 ? accd : (double)accf;
}

/* Step 16 -- SwiGLU, the activation the MLP applies between its projections
 * (named in the "future directions" section of the page): the down
 * projection reads H = silu(G) * U, elementwise over the gate product G and
 * the up product U, with silu(z) = z / (1 + e^-z).  Double precision. */
void or_swiglu(const double *G, const double *U, int64_t n, double *H)
{
    for (int64_t i = 0; i < n; i++) {
        double z = G[i];
        H[i] = z / (1.0 + exp(-z)) * U[i];
    }
}
