/*
 * entro_oracle.c -- TEST INFRASTRUCTURE, not part of the product.
 *
 * A plain, slow, obviously correct CPU restatement of what the Huffman
 * weight-compression path computes.  Only the test suite, the smoke check and
 * the benchmark's CPU-baseline leg may load it.  It shares no code, header or
 * table with the CUDA library and never looks at a decoding table: every
 * decode walks the canonical code one bit at a time.
 *
 * What it follows:
 *  - Tensor-level mixed quantization, unsigned or asymmetric per tensor:
 *    "EntroLLM: Entropy Encoded Weight Compression for Efficient Large Language
 *    Model Inference on Edge Devices" (arXiv 2505.02380v4), abstract and
 *    method details ("key design" item 1); technical summary on gist.science,
 *    "Methodologie" item 1.  The formula scale = (max-min)/(2^b-1),
 *    zero = round(-min/scale) is the asymmetric case of that scheme.
 *  - Huffman coding of the quantized codes from their histogram: same pages,
 *    "key design" item 2 / "Methodologie" item 2.  Code lengths are limited to
 *    Lmax with the package-merge algorithm (Larmore & Hirschberg, "A fast
 *    algorithm for optimal length-limited Huffman codes", J. ACM 1990) and
 *    made canonical as in RFC 1951 section 3.2.2.
 *  - Chunked storage so chunks decode independently: EntroLLM "Methodologie"
 *    item 3 (parallel decoding over chunks); lane interleaving: "LazyWeights:
 *    Decode-on-Demand Edge LLMs" (arXiv 2611.17108v1), abstract ("Huffman-codes
 *    them losslessly in interleaved lanes").
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - all rounding to integers is round-half-to-even in double precision;
 *  - unsigned quantization is eligible only for tensors with min >= 0;
 *  - the mixed choice picks the lower empirical code entropy, ties -> unsigned;
 *  - a constant tensor quantizes to one code (0 if the value is 0, else 1
 *    with scale = the value);
 *  - package-merge ties: leaves sorted by (count, symbol); at equal weight a
 *    leaf precedes a package; a one-symbol alphabet gets length 1;
 *  - codes are written MSB-first into 32-bit words;
 *  - lane layout: L lanes (32 or 64, a format parameter), lane l holds runs
 *    of 8 consecutive symbols at chunk positions 8*L*t + 8*l + (0..7), each
 *    lane padded to the chunk's longest lane, word j of lane l stored at
 *    chunk_word_base + L*j + l.
 *  - row-tile layout (a second reading of "interleaved lanes", for the fused
 *    matrix-vector product): the tensor is cut into tiles of L rows by
 *    Kc = chunk_symbols / L columns (row groups outer, column tiles inner);
 *    lane l of a tile codes row l of the tile, its Kc (fewer in the last
 *    column tile) codes in column order; a tile with fewer than L rows leaves
 *    the remaining lanes empty.  Lanes are padded and word-interleaved as
 *    above.  Columns and Kc must be multiples of 8.
 *  - consumption-order row tiles: the same tiles and lane streams, each lane
 *    keeping only its own words, stored in the order a lock-step reference
 *    decoder takes them (section 5b).
 *
 * Numeric formulas checked elsewhere against independent pins (see tests).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_EINVAL -1
#define OR_ELIMIT -2
#define OR_EFORMAT -3
#define OR_ECORRUPT -4
#define OR_ENOMEM -5

#define OR_MODE_AUTO 0
#define OR_MODE_UNSIGNED 1
#define OR_MODE_ASYM 2

#define OR_SCHEME_UNSIGNED 0
#define OR_SCHEME_ASYM 1

#define OR_FMT_SINGLE 1
#define OR_FMT_LANES 2
#define OR_FMT_ROWS 3
#define OR_FMT_ROWS_CO 4

#define OR_RUN 8
#define OR_HEADER_BYTES 128
#define OR_LENGTHS_BYTES 256
#define OR_MAX_ZERO 16777216.0 /* |zero| <= 2^24 keeps q - zero exact in fp32 */

/* ------------------------------------------------------------------ */
/* little-endian field access (the blob is little-endian by definition) */

static void put_u32(uint8_t *p, uint32_t v) {
    for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static void put_u64(uint8_t *p, uint64_t v) {
    for (int i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static uint32_t get_u32(const uint8_t *p) {
    uint32_t v = 0;
    for (int i = 0; i < 4; i++) v |= (uint32_t)p[i] << (8 * i);
    return v;
}
static uint64_t get_u64(const uint8_t *p) {
    uint64_t v = 0;
    for (int i = 0; i < 8; i++) v |= (uint64_t)p[i] << (8 * i);
    return v;
}

/* ------------------------------------------------------------------ */
/* 1. Quantization (EntroLLM abstract: unsigned and asymmetric, tensor level) */

static double clamp_d(double v, double lo, double hi) {
    if (v < lo) return lo;
    if (v > hi) return hi;
    return v;
}

/* Shannon entropy of a code histogram, in bits per symbol. */
double or_entropy(const int64_t *hist, int nsym) {
    int64_t n = 0;
    for (int i = 0; i < nsym; i++) n += hist[i];
    if (n == 0) return 0.0;
    double h = 0.0;
    for (int i = 0; i < nsym; i++) {
        if (hist[i] > 0) {
            double p = (double)hist[i] / (double)n;
            h -= p * log2(p);
        }
    }
    return h;
}

void or_histogram(const uint8_t *q, int64_t n, int nsym, int64_t *hist) {
    for (int i = 0; i < nsym; i++) hist[i] = 0;
    for (int64_t i = 0; i < n; i++) hist[q[i]] += 1;
}

/* Unsigned: zero = 0, scale = max / (2^b - 1); needs min >= 0 and max > 0. */
static int quant_unsigned(const float *w, int64_t n, int qmax, float mx, uint8_t *q, float *s) {
    float scale = (float)((double)mx / (double)qmax);
    if (!(scale > 0.0f) || isinf(scale)) return OR_ELIMIT;
    for (int64_t i = 0; i < n; i++) {
        double v = nearbyint((double)w[i] / (double)scale);
        q[i] = (uint8_t)clamp_d(v, 0.0, (double)qmax);
    }
    *s = scale;
    return OR_OK;
}

/* Asymmetric: scale = (max - min) / (2^b - 1), zero = round(-min / scale),
 * q = clamp(round(w / scale) + zero, 0, 2^b - 1). */
static int quant_asym(const float *w, int64_t n, int qmax, float mn, float mx,
                      uint8_t *q, float *s, int32_t *z) {
    float scale = (float)(((double)mx - (double)mn) / (double)qmax);
    if (!(scale > 0.0f) || isinf(scale)) return OR_ELIMIT;
    double zero = nearbyint(-(double)mn / (double)scale);
    if (fabs(zero) > OR_MAX_ZERO) return OR_ELIMIT;
    for (int64_t i = 0; i < n; i++) {
        double v = nearbyint((double)w[i] / (double)scale) + zero;
        q[i] = (uint8_t)clamp_d(v, 0.0, (double)qmax);
    }
    *s = scale;
    *z = (int32_t)zero;
    return OR_OK;
}

int or_quantize(const float *w, int64_t n, int bits, int mode, uint8_t *q,
                float *scale, int32_t *zero, int32_t *scheme) {
    if ((bits != 4 && bits != 8) || mode < 0 || mode > 2 || n < 0) return OR_EINVAL;
    int qmax = (1 << bits) - 1;
    *zero = 0;
    *scale = 1.0f;
    *scheme = (mode == OR_MODE_ASYM) ? OR_SCHEME_ASYM : OR_SCHEME_UNSIGNED;
    if (n == 0) return OR_OK;
    for (int64_t i = 0; i < n; i++)
        if (!isfinite(w[i])) return OR_EINVAL;
    float mn = w[0], mx = w[0];
    for (int64_t i = 1; i < n; i++) {
        if (w[i] < mn) mn = w[i];
        if (w[i] > mx) mx = w[i];
    }
    if (mode == OR_MODE_UNSIGNED && mn < 0.0f) return OR_EINVAL;

    if (mx == mn) { /* constant tensor: one code */
        if (mode == OR_MODE_AUTO) *scheme = (mn >= 0.0f) ? OR_SCHEME_UNSIGNED : OR_SCHEME_ASYM;
        uint8_t code = (mn == 0.0f) ? 0 : 1;
        *scale = (mn == 0.0f) ? 1.0f : mn;
        for (int64_t i = 0; i < n; i++) q[i] = code;
        return OR_OK;
    }

    if (mode == OR_MODE_UNSIGNED) {
        *scheme = OR_SCHEME_UNSIGNED;
        return quant_unsigned(w, n, qmax, mx, q, scale);
    }
    if (mode == OR_MODE_ASYM) {
        *scheme = OR_SCHEME_ASYM;
        return quant_asym(w, n, qmax, mn, mx, q, scale, zero);
    }

    /* AUTO: both candidates, keep the one whose codes have lower entropy. */
    uint8_t *qa = (uint8_t *)malloc((size_t)n);
    if (!qa) return OR_ENOMEM;
    float sa = 0.0f;
    int32_t za = 0;
    int ra = quant_asym(w, n, qmax, mn, mx, qa, &sa, &za);
    int ru = OR_EINVAL;
    float su = 0.0f;
    if (mn >= 0.0f) ru = quant_unsigned(w, n, qmax, mx, q, &su);
    if (ru != OR_OK && ra != OR_OK) {
        free(qa);
        return ra;
    }
    int take_unsigned;
    if (ru != OR_OK) {
        take_unsigned = 0;
    } else if (ra != OR_OK) {
        take_unsigned = 1;
    } else {
        int64_t hu[256], ha[256];
        or_histogram(q, n, qmax + 1, hu);
        or_histogram(qa, n, qmax + 1, ha);
        double eu = or_entropy(hu, qmax + 1), ea = or_entropy(ha, qmax + 1);
        take_unsigned = (eu <= ea + 1e-9);
    }
    if (take_unsigned) {
        *scheme = OR_SCHEME_UNSIGNED;
        *scale = su;
        *zero = 0;
    } else {
        *scheme = OR_SCHEME_ASYM;
        *scale = sa;
        *zero = za;
        memcpy(q, qa, (size_t)n);
    }
    free(qa);
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* 2. Length-limited code lengths by package-merge (coin-collector form).
 *
 * Every item carries its weight and how many times each symbol's leaf occurs
 * inside it.  list(Lmax) = the leaves; list(d) = merge(leaves, pairs of
 * list(d+1)) for d = Lmax-1 .. 1.  The 2m-2 lightest items of list(1) are
 * selected and a symbol's code length is its leaf count over them. */

typedef struct {
    int64_t weight;
    int is_leaf;
    uint16_t *cnt; /* per-symbol leaf occurrences, nsym entries */
} pm_item;

static int leaf_less(const int64_t *hist, int a, int b) {
    if (hist[a] != hist[b]) return hist[a] < hist[b];
    return a < b;
}

int or_code_lengths(const int64_t *hist, int nsym, int max_len, uint8_t *len) {
    if (nsym < 1 || nsym > 256 || max_len < 1 || max_len > 24) return OR_EINVAL;
    int syms[256], m = 0;
    for (int i = 0; i < nsym; i++) {
        len[i] = 0;
        if (hist[i] < 0) return OR_EINVAL;
        if (hist[i] > 0) syms[m++] = i;
    }
    if (m == 0) return OR_OK;
    if (m == 1) {
        len[syms[0]] = 1;
        return OR_OK;
    }
    if (max_len < 31 && (int64_t)m > ((int64_t)1 << max_len)) return OR_ELIMIT;
    /* leaves sorted by (count ascending, symbol ascending): insertion sort */
    for (int i = 1; i < m; i++) {
        int v = syms[i], j = i - 1;
        while (j >= 0 && leaf_less(hist, v, syms[j])) {
            syms[j + 1] = syms[j];
            j--;
        }
        syms[j + 1] = v;
    }
    int cap = 2 * m;
    pm_item *cur = (pm_item *)calloc((size_t)cap, sizeof(pm_item));
    pm_item *nxt = (pm_item *)calloc((size_t)cap, sizeof(pm_item));
    uint16_t *pool_a = (uint16_t *)calloc((size_t)cap * nsym, sizeof(uint16_t));
    uint16_t *pool_b = (uint16_t *)calloc((size_t)cap * nsym, sizeof(uint16_t));
    uint16_t *pkg = (uint16_t *)calloc((size_t)m * nsym, sizeof(uint16_t));
    int64_t *pkg_w = (int64_t *)calloc((size_t)m, sizeof(int64_t));
    if (!cur || !nxt || !pool_a || !pool_b || !pkg || !pkg_w) {
        free(cur); free(nxt); free(pool_a); free(pool_b); free(pkg); free(pkg_w);
        return OR_ENOMEM;
    }
    for (int i = 0; i < cap; i++) {
        cur[i].cnt = pool_a + (size_t)i * nsym;
        nxt[i].cnt = pool_b + (size_t)i * nsym;
    }
    int ncur = m;
    for (int i = 0; i < m; i++) {
        cur[i].weight = hist[syms[i]];
        cur[i].is_leaf = 1;
        memset(cur[i].cnt, 0, sizeof(uint16_t) * nsym);
        cur[i].cnt[syms[i]] = 1;
    }
    for (int d = max_len - 1; d >= 1; d--) {
        /* package consecutive pairs of the current list */
        int np = ncur / 2;
        for (int p = 0; p < np; p++) {
            pkg_w[p] = cur[2 * p].weight + cur[2 * p + 1].weight;
            for (int s = 0; s < nsym; s++)
                pkg[(size_t)p * nsym + s] = (uint16_t)(cur[2 * p].cnt[s] + cur[2 * p + 1].cnt[s]);
        }
        /* merge the leaves with the packages; a leaf goes first on equal weight */
        int li = 0, pi = 0, k = 0;
        while (li < m || pi < np) {
            int take_leaf;
            if (li >= m) take_leaf = 0;
            else if (pi >= np) take_leaf = 1;
            else take_leaf = hist[syms[li]] <= pkg_w[pi];
            if (take_leaf) {
                nxt[k].weight = hist[syms[li]];
                nxt[k].is_leaf = 1;
                memset(nxt[k].cnt, 0, sizeof(uint16_t) * nsym);
                nxt[k].cnt[syms[li]] = 1;
                li++;
            } else {
                nxt[k].weight = pkg_w[pi];
                nxt[k].is_leaf = 0;
                memcpy(nxt[k].cnt, pkg + (size_t)pi * nsym, sizeof(uint16_t) * nsym);
                pi++;
            }
            k++;
        }
        pm_item *t = cur;
        cur = nxt;
        nxt = t;
        ncur = k;
    }
    int take = 2 * m - 2;
    int status = OR_OK;
    if (take > ncur) {
        status = OR_ELIMIT;
    } else {
        int acc[256] = {0};
        for (int i = 0; i < take; i++)
            for (int s = 0; s < nsym; s++) acc[s] += cur[i].cnt[s];
        for (int s = 0; s < nsym; s++) len[s] = (uint8_t)acc[s];
    }
    free(cur); free(nxt); free(pool_a); free(pool_b); free(pkg); free(pkg_w);
    return status;
}

/* ------------------------------------------------------------------ */
/* 3. Canonical codes (RFC 1951 section 3.2.2). */

int or_canonical_codes(const uint8_t *len, int nsym, uint32_t *code) {
    int bl_count[33] = {0};
    uint32_t next_code[33] = {0};
    for (int s = 0; s < nsym; s++) {
        if (len[s] > 32) return OR_EINVAL;
        bl_count[len[s]]++;
    }
    bl_count[0] = 0;
    uint32_t c = 0;
    for (int b = 1; b <= 32; b++) {
        c = (c + (uint32_t)bl_count[b - 1]) << 1;
        next_code[b] = c;
    }
    for (int s = 0; s < nsym; s++) {
        code[s] = 0;
        if (len[s] != 0) code[s] = next_code[len[s]]++;
    }
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* 4. Bit writer / reader: MSB-first inside 32-bit words. */

typedef struct {
    uint32_t *words; /* NULL: count only */
    uint64_t nbits;
} bitw;

static void put_bit(bitw *bw, int bit) {
    if (bw->words && bit) bw->words[bw->nbits >> 5] |= 1u << (31 - (bw->nbits & 31));
    bw->nbits++;
}

static void put_code(bitw *bw, uint32_t code, int length) {
    for (int i = length - 1; i >= 0; i--) put_bit(bw, (int)((code >> i) & 1u));
}

/* ------------------------------------------------------------------ */
/* 5. Encoder: quantize -> histogram -> lengths -> canonical codes -> chunks.
 *
 * Blob (little-endian):
 *   [0,128)   header: magic "ENTR", version 1, bits, scheme, max_len, format,
 *             lanes, run, rows, cols, n, chunk_symbols, n_chunks, scale (fp32
 *             bits), zero (int32), payload_words, zero padding
 *   [128,384) code length of each of the 256 symbols (0 = unused)
 *   index     (n_chunks + 1) x {u64 start, u64 first_symbol}; start is a bit
 *             offset (single stream) or a word offset (lanes)
 *   payload   payload_words x u32
 */

/* Row-tile layout: tiles of `lanes` rows by kc = chunk_symbols / lanes
 * columns, row groups outer and column tiles inner; chunk c is one tile. */
typedef struct {
    int64_t row0, col0; /* first row and column of the tile */
    int nrows;          /* rows in the tile (lanes that hold codes) */
    int64_t width;      /* columns in the tile */
    uint64_t first;     /* symbols in all earlier tiles */
} tile;

static uint64_t rows_tiles(int64_t rows, int64_t cols, int lanes, int64_t chunk_symbols) {
    if (rows <= 0 || cols <= 0) return 0;
    int64_t kc = chunk_symbols / lanes;
    return (uint64_t)((rows + lanes - 1) / lanes) * (uint64_t)((cols + kc - 1) / kc);
}

static tile tile_of(int64_t rows, int64_t cols, int lanes, int64_t chunk_symbols, uint64_t c) {
    int64_t kc = chunk_symbols / lanes;
    int64_t tiles_per_group = (cols + kc - 1) / kc;
    int64_t g = (int64_t)c / tiles_per_group, j = (int64_t)c % tiles_per_group;
    tile t;
    t.row0 = g * lanes;
    t.col0 = j * kc;
    t.nrows = (int)(rows - t.row0 < lanes ? rows - t.row0 : lanes);
    t.width = cols - t.col0 < kc ? cols - t.col0 : kc;
    t.first = (uint64_t)(t.row0 * cols + (int64_t)t.nrows * t.col0);
    return t;
}

/* ------------------------------------------------------------------ */
/* 5b. Row tiles in consumption order (format 4).
 *
 * A tile's lanes code the same bits as in the row-tile layout; what differs
 * is where their words sit.  Word-by-word interleaving pads every lane to the
 * tile's longest lane; here a lane keeps only its own words, and after its
 * first three they are stored in the order a reference decoder running all
 * lanes in lock step takes them.  A chunk is
 *   [the number of words of each lane: L counts of 1 byte, or of 2 bytes
 *    when ceil(Kc * max_len / 32) > 255, little-endian, zero-padded to whole
 *    words]
 *   [words 0, 1, 2 of every lane, word j of lane l at row j, column l (zero
 *    where the lane has fewer words)]
 *   [every later word, in the order the reference decoder takes them]
 *   [zero words up to a multiple of 4 words]
 * The reference decoder, per lane:
 *   - a lookup takes, from the lane's next codes, the longest run of whole
 *     codes whose lengths add up to at most 12 bits, at most 8 codes (4-bit)
 *     or 4 (8-bit); when the next code is longer than 12 bits it takes that
 *     code alone;
 *   - lookups are numbered 0, 1, 2, ...; a refill point comes before each
 *     even-numbered lookup (before every lookup when the code length limit
 *     max_len is above 16);
 *   - the lane adds the bits of each lookup to a count c (0 at the start); at
 *     a refill point with c >= 32 it subtracts 32 and, if some of its words
 *     are not yet placed, takes the next one;
 *   - the words taken at one refill point are placed in lane order.
 */
#define OR_PEEK_BITS 12

static int co_count_bytes(int64_t kc, int max_len) { return ((int64_t)kc * max_len + 31) / 32 <= 255 ? 1 : 2; }

static uint64_t co_header_words(int lanes, int count_bytes) { return ((uint64_t)lanes * (uint64_t)count_bytes + 3) / 4; }

typedef struct {
    int64_t width;      /* codes of the lane */
    int64_t done;       /* codes its lookups have taken */
    int64_t lookups;    /* lookups made */
    int c;              /* bits taken since the start, less 32 per refill */
    uint64_t nw, taken; /* words of the lane; words placed so far */
} co_lane;

/* length of code i of a lane (decoding it first if needed), < 0 on error */
typedef int (*co_len_fn)(void *ctx, int lane, int64_t i);
/* word `word` of a lane is the next one placed */
typedef int (*co_place_fn)(void *ctx, int lane, uint64_t word);

/* Replay the reference decoder over the lanes of one tile, calling place()
 * for each word after a lane's first three, in placement order. */
static int co_schedule(co_lane *ln, int lanes, int every, int bits, co_len_fn len_of, co_place_fn place,
                       void *ctx) {
    const int m = bits == 4 ? 8 : 4;
    for (uint64_t p = 0;; p++) {
        int open = 0;
        for (int l = 0; l < lanes; l++) {
            co_lane *s = &ln[l];
            if (s->taken >= s->nw) continue;
            open = 1;
            const int64_t before = every ? (int64_t)p : 2 * (int64_t)p; /* lookups before this refill point */
            while (s->lookups < before) {
                if (s->done >= s->width) return OR_ECORRUPT; /* words left but no codes */
                int first = len_of(ctx, l, s->done);
                if (first < 0) return first;
                int used = 0;
                int64_t k = 0;
                if (first > OR_PEEK_BITS) {
                    used = first;
                    k = 1;
                } else {
                    while (k < m && s->done + k < s->width) {
                        int lk = len_of(ctx, l, s->done + k);
                        if (lk < 0) return lk;
                        if (used + lk > OR_PEEK_BITS) break;
                        used += lk;
                        k++;
                    }
                }
                s->done += k;
                s->c += used;
                s->lookups++;
            }
            if (s->c >= 32) {
                s->c -= 32;
                int r = place(ctx, l, s->taken);
                if (r != OR_OK) return r;
                s->taken++;
            }
        }
        if (!open) return OR_OK;
    }
}

/* encoder side: the lanes' code lengths are known */
typedef struct {
    const uint8_t *const *lens; /* per lane, code lengths in column order */
    uint32_t *const *words;     /* per lane, its words */
    uint32_t *out;              /* the chunk's words */
    uint64_t pos;               /* next placement */
} co_enc;

static int co_enc_len(void *ctx, int lane, int64_t i) { return ((co_enc *)ctx)->lens[lane][i]; }

static int co_enc_place(void *ctx, int lane, uint64_t word) {
    co_enc *e = (co_enc *)ctx;
    e->out[e->pos++] = e->words[lane][word];
    return OR_OK;
}

/* words of one consumption-order tile (header, three rows, the rest, padding) */
static uint64_t co_tile_words(const uint64_t *nw, int lanes, int count_bytes) {
    uint64_t w = co_header_words(lanes, count_bytes) + 3 * (uint64_t)lanes;
    for (int l = 0; l < lanes; l++) w += nw[l] > 3 ? nw[l] - 3 : 0;
    return (w + 3) & ~(uint64_t)3;
}

int or_encode(const float *w, int64_t rows, int64_t cols, int bits, int mode, int max_len,
              int format, int64_t chunk_symbols, int lanes, uint8_t *out, uint64_t cap, uint64_t *out_size) {
    if (rows < 0 || cols < 0 || (bits != 4 && bits != 8)) return OR_EINVAL;
    if (format != OR_FMT_SINGLE && format != OR_FMT_LANES && format != OR_FMT_ROWS && format != OR_FMT_ROWS_CO)
        return OR_EINVAL;
    const int tiles = format == OR_FMT_ROWS || format == OR_FMT_ROWS_CO;
    if (max_len == 0) max_len = (bits == 8) ? 16 : 12;
    if (max_len < 1 || max_len > 24) return OR_EINVAL;
    if (chunk_symbols == 0) chunk_symbols = (format == OR_FMT_SINGLE) ? 4096 : 8192;
    if (format == OR_FMT_SINGLE && (chunk_symbols < 1 || chunk_symbols > (1 << 20))) return OR_EINVAL;
    if (format != OR_FMT_SINGLE && lanes == 0) lanes = 32;
    if (format != OR_FMT_SINGLE && lanes != 32 && lanes != 64) return OR_EINVAL;
    const int64_t step = (int64_t)OR_RUN * lanes; /* symbols per lane step */
    if (format != OR_FMT_SINGLE &&
        (chunk_symbols < step || chunk_symbols > 16384 || chunk_symbols % step != 0))
        return OR_EINVAL;
    if (tiles && cols % OR_RUN != 0) return OR_EINVAL;
    int64_t n = rows * cols;
    int nsym = 1 << bits;

    uint8_t *q = (uint8_t *)malloc(n > 0 ? (size_t)n : 1);
    if (!q) return OR_ENOMEM;
    float scale;
    int32_t zero, scheme;
    int r = or_quantize(w, n, bits, mode, q, &scale, &zero, &scheme);
    if (r != OR_OK) { free(q); return r; }

    int64_t hist[256];
    or_histogram(q, n, nsym, hist);
    uint8_t len[256];
    memset(len, 0, sizeof(len));
    r = or_code_lengths(hist, nsym, max_len, len);
    if (r != OR_OK) { free(q); return r; }
    uint32_t code[256];
    or_canonical_codes(len, 256, code);

    uint64_t n_chunks = n > 0 ? (uint64_t)((n + chunk_symbols - 1) / chunk_symbols) : 0;
    if (tiles) n_chunks = rows_tiles(rows, cols, lanes, chunk_symbols);
    const int count_bytes = co_count_bytes(chunk_symbols / lanes, max_len);
    const int every = max_len > 16;

    /* pass 1: sizes.  Single stream: total bits.  Lanes: per-chunk word count. */
    uint64_t *start = (uint64_t *)calloc(n_chunks + 1, sizeof(uint64_t));
    if (!start) { free(q); return OR_ENOMEM; }
    uint64_t payload_words = 0;
    if (format == OR_FMT_SINGLE) {
        uint64_t bitpos = 0;
        for (uint64_t c = 0; c < n_chunks; c++) {
            start[c] = bitpos;
            uint64_t a = c * (uint64_t)chunk_symbols, b = a + (uint64_t)chunk_symbols;
            if (b > (uint64_t)n) b = (uint64_t)n;
            for (uint64_t i = a; i < b; i++) bitpos += len[q[i]];
        }
        start[n_chunks] = bitpos;
        payload_words = (bitpos + 31) / 32;
    } else if (format == OR_FMT_ROWS_CO) {
        uint64_t wpos = 0, nw[64];
        for (uint64_t c = 0; c < n_chunks; c++) {
            start[c] = wpos;
            tile t = tile_of(rows, cols, lanes, chunk_symbols, c);
            for (int l = 0; l < lanes; l++) {
                uint64_t lane_bits = 0;
                if (l < t.nrows)
                    for (int64_t k = 0; k < t.width; k++) lane_bits += len[q[(t.row0 + l) * cols + t.col0 + k]];
                nw[l] = (lane_bits + 31) / 32;
            }
            wpos += co_tile_words(nw, lanes, count_bytes);
        }
        start[n_chunks] = wpos;
        payload_words = wpos;
    } else if (format == OR_FMT_ROWS) {
        uint64_t wpos = 0;
        for (uint64_t c = 0; c < n_chunks; c++) {
            start[c] = wpos;
            tile t = tile_of(rows, cols, lanes, chunk_symbols, c);
            uint64_t wmax = 0;
            for (int l = 0; l < t.nrows; l++) {
                uint64_t lane_bits = 0;
                for (int64_t k = 0; k < t.width; k++) lane_bits += len[q[(t.row0 + l) * cols + t.col0 + k]];
                uint64_t wl = (lane_bits + 31) / 32;
                if (wl > wmax) wmax = wl;
            }
            wpos += wmax * (uint64_t)lanes;
        }
        start[n_chunks] = wpos;
        payload_words = wpos;
    } else {
        uint64_t wpos = 0;
        for (uint64_t c = 0; c < n_chunks; c++) {
            start[c] = wpos;
            uint64_t a = c * (uint64_t)chunk_symbols, b = a + (uint64_t)chunk_symbols;
            if (b > (uint64_t)n) b = (uint64_t)n;
            uint64_t nc = b - a, wmax = 0;
            for (int l = 0; l < lanes; l++) {
                uint64_t lane_bits = 0;
                for (uint64_t p = 0; p < nc; p++)
                    if ((p % (uint64_t)step) / OR_RUN == (uint64_t)l) lane_bits += len[q[a + p]];
                uint64_t wl = (lane_bits + 31) / 32;
                if (wl > wmax) wmax = wl;
            }
            wpos += wmax * (uint64_t)lanes;
        }
        start[n_chunks] = wpos;
        payload_words = wpos;
    }

    uint64_t index_bytes = 16 * (n_chunks + 1);
    uint64_t total = OR_HEADER_BYTES + OR_LENGTHS_BYTES + index_bytes + 4 * payload_words;
    *out_size = total;
    if (out == NULL || cap < total) { free(q); free(start); return OR_OK; }

    memset(out, 0, (size_t)total);
    put_u32(out + 0, 0x52544E45u);
    put_u32(out + 4, 1);
    put_u32(out + 8, (uint32_t)bits);
    put_u32(out + 12, (uint32_t)scheme);
    put_u32(out + 16, (uint32_t)max_len);
    put_u32(out + 20, (uint32_t)format);
    put_u32(out + 24, format == OR_FMT_SINGLE ? 1u : (uint32_t)lanes);  /* lanes or rows per tile */
    put_u32(out + 28, format == OR_FMT_SINGLE ? 1u : (uint32_t)OR_RUN);
    put_u64(out + 32, (uint64_t)rows);
    put_u64(out + 40, (uint64_t)cols);
    put_u64(out + 48, (uint64_t)n);
    put_u64(out + 56, (uint64_t)chunk_symbols);
    put_u64(out + 64, n_chunks);
    uint32_t sbits;
    memcpy(&sbits, &scale, 4);
    put_u32(out + 72, sbits);
    put_u32(out + 76, (uint32_t)zero);
    put_u64(out + 80, payload_words);
    memcpy(out + OR_HEADER_BYTES, len, 256);
    uint8_t *idx = out + OR_HEADER_BYTES + OR_LENGTHS_BYTES;
    for (uint64_t c = 0; c <= n_chunks; c++) {
        uint64_t first = c * (uint64_t)chunk_symbols;
        if (tiles) first = c < n_chunks ? tile_of(rows, cols, lanes, chunk_symbols, c).first : (uint64_t)n;
        if (first > (uint64_t)n) first = (uint64_t)n;
        put_u64(idx + 16 * c, start[c]);
        put_u64(idx + 16 * c + 8, first);
    }

    /* pass 2: the bits */
    uint32_t *payload = (uint32_t *)calloc(payload_words ? payload_words : 1, sizeof(uint32_t));
    if (!payload) { free(q); free(start); return OR_ENOMEM; }
    if (format == OR_FMT_SINGLE) {
        bitw bw = {payload, 0};
        for (int64_t i = 0; i < n; i++) put_code(&bw, code[q[i]], len[q[i]]);
    } else if (format == OR_FMT_ROWS_CO) {
        const int64_t kc = chunk_symbols / lanes;
        const uint64_t max_words = ((uint64_t)kc * (uint64_t)max_len + 31) / 32;
        uint32_t *lw[64];
        uint8_t *ll[64];
        uint64_t nw[64];
        int rc = OR_OK;
        for (int l = 0; l < lanes; l++) {
            lw[l] = (uint32_t *)calloc(max_words + 1, sizeof(uint32_t));
            ll[l] = (uint8_t *)malloc((size_t)kc);
            if (!lw[l] || !ll[l]) rc = OR_ENOMEM;
        }
        for (uint64_t c = 0; rc == OR_OK && c < n_chunks; c++) {
            tile t = tile_of(rows, cols, lanes, chunk_symbols, c);
            co_lane st[64];
            for (int l = 0; l < lanes; l++) {
                memset(lw[l], 0, sizeof(uint32_t) * (max_words + 1));
                bitw bw = {lw[l], 0};
                int64_t width = l < t.nrows ? t.width : 0;
                for (int64_t k = 0; k < width; k++) {
                    uint8_t v = q[(t.row0 + l) * cols + t.col0 + k];
                    put_code(&bw, code[v], len[v]);
                    ll[l][k] = len[v];
                }
                nw[l] = (bw.nbits + 31) / 32;
                st[l].width = width;
                st[l].done = st[l].lookups = 0;
                st[l].c = 0;
                st[l].nw = nw[l];
                st[l].taken = nw[l] < 3 ? nw[l] : 3;
            }
            uint32_t *chunk = payload + start[c];
            /* counts, little-endian, count_bytes each */
            uint8_t *hdr = (uint8_t *)chunk;
            for (int l = 0; l < lanes; l++) {
                hdr[count_bytes * l] = (uint8_t)(nw[l] & 0xFF);
                if (count_bytes == 2) hdr[2 * l + 1] = (uint8_t)(nw[l] >> 8);
            }
            /* the header bytes were written into host-order words: make them little-endian words */
            const uint64_t hw = co_header_words(lanes, count_bytes);
            for (uint64_t j = 0; j < hw; j++) chunk[j] = get_u32(hdr + 4 * j);
            for (int j = 0; j < 3; j++)
                for (int l = 0; l < lanes; l++) chunk[hw + (uint64_t)lanes * j + l] = (uint64_t)j < nw[l] ? lw[l][j] : 0;
            co_enc e = {(const uint8_t *const *)ll, (uint32_t *const *)lw, chunk, hw + 3 * (uint64_t)lanes};
            rc = co_schedule(st, lanes, every, bits, co_enc_len, co_enc_place, &e);
            if (rc == OR_OK && start[c] + e.pos > start[c + 1]) rc = OR_EINVAL;
        }
        for (int l = 0; l < lanes; l++) { free(lw[l]); free(ll[l]); }
        if (rc != OR_OK) { free(q); free(start); free(payload); return rc; }
    } else if (format == OR_FMT_ROWS) {
        for (uint64_t c = 0; c < n_chunks; c++) {
            tile t = tile_of(rows, cols, lanes, chunk_symbols, c);
            uint64_t wmax = (start[c + 1] - start[c]) / (uint64_t)lanes;
            uint32_t *lane_words = (uint32_t *)calloc(wmax ? wmax : 1, sizeof(uint32_t));
            if (!lane_words) { free(q); free(start); free(payload); return OR_ENOMEM; }
            for (int l = 0; l < t.nrows; l++) {
                memset(lane_words, 0, sizeof(uint32_t) * (wmax ? wmax : 1));
                bitw bw = {lane_words, 0};
                for (int64_t k = 0; k < t.width; k++) {
                    uint8_t v = q[(t.row0 + l) * cols + t.col0 + k];
                    put_code(&bw, code[v], len[v]);
                }
                for (uint64_t j = 0; j < wmax; j++) payload[start[c] + (uint64_t)lanes * j + l] = lane_words[j];
            }
            free(lane_words);
        }
    } else {
        for (uint64_t c = 0; c < n_chunks; c++) {
            uint64_t a = c * (uint64_t)chunk_symbols, b = a + (uint64_t)chunk_symbols;
            if (b > (uint64_t)n) b = (uint64_t)n;
            uint64_t nc = b - a;
            uint64_t wmax = (start[c + 1] - start[c]) / (uint64_t)lanes;
            uint32_t *lane_words = (uint32_t *)calloc(wmax ? wmax : 1, sizeof(uint32_t));
            if (!lane_words) { free(q); free(start); free(payload); return OR_ENOMEM; }
            for (int l = 0; l < lanes; l++) {
                memset(lane_words, 0, sizeof(uint32_t) * (wmax ? wmax : 1));
                bitw bw = {lane_words, 0};
                for (uint64_t p = 0; p < nc; p++)
                    if ((p % (uint64_t)step) / OR_RUN == (uint64_t)l) put_code(&bw, code[q[a + p]], len[q[a + p]]);
                for (uint64_t j = 0; j < wmax; j++) payload[start[c] + (uint64_t)lanes * j + l] = lane_words[j];
            }
            free(lane_words);
        }
    }
    uint8_t *pp = idx + index_bytes;
    for (uint64_t j = 0; j < payload_words; j++) put_u32(pp + 4 * j, payload[j]);
    free(payload);
    free(start);
    free(q);
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* 6. Decoder: parse, then walk the canonical code bit by bit. */

typedef struct {
    int bits, scheme, max_len, format, lanes, run;
    uint64_t rows, cols, n, chunk_symbols, n_chunks, payload_words;
    float scale;
    int32_t zero;
    uint8_t len[256];
    const uint8_t *index;
    const uint8_t *payload;
    /* canonical description: for each length, first code, count, and the
     * symbols of that length in ascending order */
    uint32_t first[33];
    int count[33];
    int sym_by_len[33][256];
} or_blob;

static int parse(const uint8_t *blob, uint64_t size, or_blob *b) {
    if (size < OR_HEADER_BYTES + OR_LENGTHS_BYTES) return OR_EFORMAT;
    if (get_u32(blob) != 0x52544E45u || get_u32(blob + 4) != 1) return OR_EFORMAT;
    b->bits = (int)get_u32(blob + 8);
    b->scheme = (int)get_u32(blob + 12);
    b->max_len = (int)get_u32(blob + 16);
    b->format = (int)get_u32(blob + 20);
    b->lanes = (int)get_u32(blob + 24);
    b->run = (int)get_u32(blob + 28);
    b->rows = get_u64(blob + 32);
    b->cols = get_u64(blob + 40);
    b->n = get_u64(blob + 48);
    b->chunk_symbols = get_u64(blob + 56);
    b->n_chunks = get_u64(blob + 64);
    uint32_t sbits = get_u32(blob + 72);
    memcpy(&b->scale, &sbits, 4);
    b->zero = (int32_t)get_u32(blob + 76);
    b->payload_words = get_u64(blob + 80);
    if (b->bits != 4 && b->bits != 8) return OR_EFORMAT;
    if (b->format != OR_FMT_SINGLE && b->format != OR_FMT_LANES && b->format != OR_FMT_ROWS &&
        b->format != OR_FMT_ROWS_CO)
        return OR_EFORMAT;
    if (b->format != OR_FMT_SINGLE && b->lanes != 32 && b->lanes != 64) return OR_EFORMAT;
    if (b->format == OR_FMT_SINGLE && b->lanes != 1) return OR_EFORMAT;
    if (b->max_len < 1 || b->max_len > 24) return OR_EFORMAT;
    if (b->chunk_symbols == 0 || b->n != b->rows * b->cols) return OR_EFORMAT;
    if (b->format == OR_FMT_ROWS || b->format == OR_FMT_ROWS_CO) {
        if (b->chunk_symbols % (OR_RUN * (uint64_t)b->lanes) || b->cols % OR_RUN) return OR_EFORMAT;
        if (b->n_chunks != rows_tiles((int64_t)b->rows, (int64_t)b->cols, b->lanes, (int64_t)b->chunk_symbols))
            return OR_EFORMAT;
    } else if (b->n_chunks != (b->n + b->chunk_symbols - 1) / b->chunk_symbols) {
        return OR_EFORMAT;
    }
    uint64_t need = OR_HEADER_BYTES + OR_LENGTHS_BYTES + 16 * (b->n_chunks + 1) + 4 * b->payload_words;
    if (size < need) return OR_EFORMAT;
    memcpy(b->len, blob + OR_HEADER_BYTES, 256);
    b->index = blob + OR_HEADER_BYTES + OR_LENGTHS_BYTES;
    b->payload = b->index + 16 * (b->n_chunks + 1);
    for (int l = 0; l <= 32; l++) b->count[l] = 0;
    for (int s = 0; s < 256; s++) {
        if (b->len[s] > b->max_len) return OR_EFORMAT;
        if (b->len[s] && s >= (1 << b->bits)) return OR_EFORMAT;
        if (b->len[s]) b->sym_by_len[b->len[s]][b->count[b->len[s]]++] = s;
    }
    uint32_t c = 0;
    for (int l = 1; l <= 32; l++) {
        c = (c + (uint32_t)(l > 1 ? b->count[l - 1] : 0)) << 1;
        b->first[l] = c;
    }
    return OR_OK;
}

static int read_bit_single(const or_blob *b, uint64_t pos) {
    uint32_t word = get_u32(b->payload + 4 * (pos >> 5));
    return (int)((word >> (31 - (pos & 31))) & 1u);
}

/* decode one symbol; *pos advances; bit_at(pos) supplies the bits */
typedef int (*bit_fn)(const or_blob *, const void *ctx, uint64_t pos);

typedef struct {
    uint64_t word_base;
    int lane, lanes;
    uint64_t words;
} lane_ctx;

static int bit_lane(const or_blob *b, const void *ctx, uint64_t pos) {
    const lane_ctx *lc = (const lane_ctx *)ctx;
    uint64_t j = pos >> 5;
    if (j >= lc->words) return -1;
    uint32_t word = get_u32(b->payload + 4 * (lc->word_base + (uint64_t)lc->lanes * j + (uint64_t)lc->lane));
    return (int)((word >> (31 - (pos & 31))) & 1u);
}

typedef struct {
    uint64_t end;
} single_ctx;

static int bit_single(const or_blob *b, const void *ctx, uint64_t pos) {
    const single_ctx *sc = (const single_ctx *)ctx;
    if (pos >= sc->end) return -1;
    return read_bit_single(b, pos);
}

static int decode_symbol(const or_blob *b, bit_fn fn, const void *ctx, uint64_t *pos) {
    uint32_t code = 0;
    for (int l = 1; l <= b->max_len; l++) {
        int bit = fn(b, ctx, *pos);
        if (bit < 0) return OR_ECORRUPT;
        *pos += 1;
        code = (code << 1) | (uint32_t)bit;
        if (b->count[l] > 0 && code >= b->first[l] && code - b->first[l] < (uint32_t)b->count[l])
            return b->sym_by_len[l][code - b->first[l]];
    }
    return OR_ECORRUPT;
}

/* Consumption-order tile c: replay the reference decoder to find each lane's
 * words, decoding each lane's codes bit by bit as the replay needs their
 * lengths, then decode the rest of every lane. */
typedef struct {
    const or_blob *b;
    const uint8_t *chunk; /* the chunk's bytes */
    uint64_t chunk_words, pos;
    int lanes;
    uint32_t *words[64];  /* per lane: its words in order */
    uint64_t nw[64];
    uint64_t bitpos[64];  /* bits of the lane its decoded codes took */
    int64_t decoded[64];  /* codes decoded */
    uint8_t *sym[64];     /* decoded symbols */
    uint8_t *len[64];     /* their lengths */
    uint64_t have[64];    /* words of the lane known so far */
} co_dec;

typedef struct {
    const co_dec *d;
    int lane;
} co_bits;

static int bit_co(const or_blob *b, const void *ctx, uint64_t pos) {
    (void)b;
    const co_bits *cb = (const co_bits *)ctx;
    uint64_t j = pos >> 5;
    if (j >= cb->d->have[cb->lane]) return -1;
    return (int)((cb->d->words[cb->lane][j] >> (31 - (pos & 31))) & 1u);
}

static int co_dec_len(void *ctx, int lane, int64_t i) {
    co_dec *d = (co_dec *)ctx;
    while (d->decoded[lane] <= i) {
        co_bits cb = {d, lane};
        uint64_t before = d->bitpos[lane];
        int s = decode_symbol(d->b, bit_co, &cb, &d->bitpos[lane]);
        if (s < 0) return s;
        d->sym[lane][d->decoded[lane]] = (uint8_t)s;
        d->len[lane][d->decoded[lane]] = (uint8_t)(d->bitpos[lane] - before);
        d->decoded[lane]++;
    }
    return d->len[lane][i];
}

static int co_dec_place(void *ctx, int lane, uint64_t word) {
    co_dec *d = (co_dec *)ctx;
    if (d->pos >= d->chunk_words || word != d->have[lane]) return OR_ECORRUPT;
    d->words[lane][d->have[lane]++] = get_u32(d->chunk + 4 * d->pos);
    d->pos++;
    return OR_OK;
}

static int decode_tile_co(const or_blob *b, uint64_t c, uint64_t start, uint64_t next, const tile *t, uint8_t *out) {
    const int L = b->lanes;
    const int cbytes = co_count_bytes((int64_t)(b->chunk_symbols / (uint64_t)L), b->max_len);
    const uint64_t hw = co_header_words(L, cbytes);
    (void)c;
    if (next < start || next > b->payload_words || (next - start) % 4 || next - start < hw + 3 * (uint64_t)L)
        return OR_ECORRUPT;
    co_dec d;
    memset(&d, 0, sizeof(d));
    d.b = b;
    d.chunk = b->payload + 4 * start;
    d.chunk_words = next - start;
    d.lanes = L;
    d.pos = hw + 3 * (uint64_t)L;
    const uint64_t max_words = ((b->chunk_symbols / (uint64_t)L) * (uint64_t)b->max_len + 31) / 32;
    int r = OR_OK;
    co_lane st[64];
    for (int l = 0; l < L; l++) {
        uint64_t n = d.chunk[cbytes * l];
        if (cbytes == 2) n |= (uint64_t)d.chunk[2 * l + 1] << 8;
        int64_t width = l < t->nrows ? t->width : 0;
        if (n > max_words || (width == 0 && n != 0) || (width > 0 && n == 0)) r = OR_ECORRUPT;
        d.nw[l] = n;
        d.words[l] = (uint32_t *)calloc(max_words + 1, sizeof(uint32_t));
        d.sym[l] = (uint8_t *)malloc((size_t)(t->width > 0 ? t->width : 1));
        d.len[l] = (uint8_t *)malloc((size_t)(t->width > 0 ? t->width : 1));
        if (!d.words[l] || !d.sym[l] || !d.len[l]) r = OR_ENOMEM;
        if (r != OR_OK) continue;
        for (uint64_t j = 0; j < 3 && j < n; j++) d.words[l][j] = get_u32(d.chunk + 4 * (hw + (uint64_t)L * j + (uint64_t)l));
        d.have[l] = n < 3 ? n : 3;
        st[l].width = width;
        st[l].done = st[l].lookups = 0;
        st[l].c = 0;
        st[l].nw = n;
        st[l].taken = d.have[l];
    }
    if (r == OR_OK) r = co_schedule(st, L, b->max_len > 16, b->bits, co_dec_len, co_dec_place, &d);
    if (r == OR_OK && ((d.pos + 3) & ~(uint64_t)3) != d.chunk_words) r = OR_ECORRUPT;
    for (int l = 0; r == OR_OK && l < t->nrows; l++) {
        for (int64_t k = 0; r == OR_OK && k < t->width; k++) {
            int lk = co_dec_len(&d, l, k);
            if (lk < 0) r = lk;
        }
        for (int64_t k = 0; r == OR_OK && k < t->width; k++) out[(uint64_t)l * (uint64_t)t->width + (uint64_t)k] = d.sym[l][k];
    }
    for (int l = 0; l < L; l++) { free(d.words[l]); free(d.sym[l]); free(d.len[l]); }
    return r;
}

/* Chunk c of the row-tile layout into out (the tile's rows one after the
 * other, each in column order). */
static int decode_tile(const or_blob *b, uint64_t c, uint8_t *out) {
    uint64_t start = get_u64(b->index + 16 * c), next = get_u64(b->index + 16 * (c + 1));
    uint64_t first = get_u64(b->index + 16 * c + 8), last = get_u64(b->index + 16 * (c + 1) + 8);
    tile t = tile_of((int64_t)b->rows, (int64_t)b->cols, b->lanes, (int64_t)b->chunk_symbols, c);
    if (first != t.first || last != first + (uint64_t)t.nrows * (uint64_t)t.width) return OR_ECORRUPT;
    if (b->format == OR_FMT_ROWS_CO) return decode_tile_co(b, c, start, next, &t, out);
    const uint64_t L = (uint64_t)b->lanes;
    if (next < start || next > b->payload_words || (next - start) % L) return OR_ECORRUPT;
    lane_ctx lc = {start, 0, b->lanes, (next - start) / L};
    for (int l = 0; l < t.nrows; l++) {
        lc.lane = l;
        uint64_t pos = 0;
        for (int64_t k = 0; k < t.width; k++) {
            int s = decode_symbol(b, bit_lane, &lc, &pos);
            if (s < 0) return s;
            out[(uint64_t)l * (uint64_t)t.width + (uint64_t)k] = (uint8_t)s;
        }
    }
    return OR_OK;
}

static int decode_chunk(const or_blob *b, uint64_t c, uint8_t *out /* chunk-local */) {
    if (b->format == OR_FMT_ROWS || b->format == OR_FMT_ROWS_CO) return decode_tile(b, c, out);
    uint64_t start = get_u64(b->index + 16 * c), next = get_u64(b->index + 16 * (c + 1));
    uint64_t first = get_u64(b->index + 16 * c + 8), last = get_u64(b->index + 16 * (c + 1) + 8);
    if (first != c * b->chunk_symbols || last < first || last > b->n) return OR_ECORRUPT;
    uint64_t nc = last - first;
    if (b->format == OR_FMT_SINGLE) {
        if (next < start || (next + 31) / 32 > b->payload_words) return OR_ECORRUPT;
        single_ctx sc = {next};
        uint64_t pos = start;
        for (uint64_t i = 0; i < nc; i++) {
            int s = decode_symbol(b, bit_single, &sc, &pos);
            if (s < 0) return s;
            out[i] = (uint8_t)s;
        }
        if (pos != next) return OR_ECORRUPT;
    } else {
        const uint64_t L = (uint64_t)b->lanes, step = OR_RUN * L;
        if (next < start || next > b->payload_words || (next - start) % L) return OR_ECORRUPT;
        lane_ctx lc = {start, 0, b->lanes, (next - start) / L};
        for (int l = 0; l < b->lanes; l++) {
            lc.lane = l;
            uint64_t pos = 0;
            for (uint64_t p = 0; p < nc; p++) {
                if ((p % step) / OR_RUN != (uint64_t)l) continue;
                int s = decode_symbol(b, bit_lane, &lc, &pos);
                if (s < 0) return s;
                out[p] = (uint8_t)s;
            }
        }
    }
    return OR_OK;
}

int or_blob_params(const uint8_t *blob, uint64_t size, int64_t *out /* 14 entries */) {
    or_blob *b = (or_blob *)malloc(sizeof(or_blob));
    if (!b) return OR_ENOMEM;
    int r = parse(blob, size, b);
    if (r == OR_OK) {
        uint32_t sbits;
        memcpy(&sbits, &b->scale, 4);
        out[0] = b->bits; out[1] = b->scheme; out[2] = b->max_len; out[3] = b->format;
        out[4] = (int64_t)b->rows; out[5] = (int64_t)b->cols; out[6] = (int64_t)b->n;
        out[7] = (int64_t)b->chunk_symbols; out[8] = (int64_t)b->n_chunks;
        out[9] = (int64_t)sbits; out[10] = b->zero; out[11] = (int64_t)b->payload_words;
        out[12] = b->lanes; out[13] = b->run;
    }
    free(b);
    return r;
}

/* symbols in the chunks before chunk c (chunk order) */
static uint64_t chunk_first(const or_blob *b, uint64_t c) {
    if (b->format == OR_FMT_ROWS || b->format == OR_FMT_ROWS_CO)
        return c < b->n_chunks ? tile_of((int64_t)b->rows, (int64_t)b->cols, b->lanes, (int64_t)b->chunk_symbols, c).first
                               : b->n;
    uint64_t f = c * b->chunk_symbols;
    return f < b->n ? f : b->n;
}

/* decode chunks [c0, c1) into out: each chunk's codes in its own order
 * (row-major for the single-stream and lanes layouts; the tile's rows one
 * after the other for the row-tile layout), chunk c at out + (symbols in the
 * chunks c0 .. c-1) */
int or_decode_chunks(const uint8_t *blob, uint64_t size, uint64_t c0, uint64_t c1, uint8_t *out) {
    or_blob *b = (or_blob *)malloc(sizeof(or_blob));
    if (!b) return OR_ENOMEM;
    int r = parse(blob, size, b);
    if (r == OR_OK && (c0 > c1 || c1 > b->n_chunks)) r = OR_EINVAL;
    uint64_t base = r == OR_OK ? chunk_first(b, c0) : 0;
    for (uint64_t c = c0; r == OR_OK && c < c1; c++)
        r = decode_chunk(b, c, out + (chunk_first(b, c) - base));
    free(b);
    return r;
}

/* whole tensor, row-major */
int or_decode(const uint8_t *blob, uint64_t size, uint8_t *out) {
    or_blob *b = (or_blob *)malloc(sizeof(or_blob));
    if (!b) return OR_ENOMEM;
    int r = parse(blob, size, b);
    if (r != OR_OK || (b->format != OR_FMT_ROWS && b->format != OR_FMT_ROWS_CO)) {
        uint64_t nch = b->n_chunks;
        free(b);
        if (r != OR_OK) return r;
        return or_decode_chunks(blob, size, 0, nch, out);
    }
    /* row tiles: decode each tile, then place its rows */
    uint8_t *tmp = (uint8_t *)malloc((size_t)b->chunk_symbols);
    if (!tmp) { free(b); return OR_ENOMEM; }
    for (uint64_t c = 0; r == OR_OK && c < b->n_chunks; c++) {
        tile t = tile_of((int64_t)b->rows, (int64_t)b->cols, b->lanes, (int64_t)b->chunk_symbols, c);
        r = decode_tile(b, c, tmp);
        for (int l = 0; r == OR_OK && l < t.nrows; l++)
            memcpy(out + (uint64_t)(t.row0 + l) * b->cols + (uint64_t)t.col0, tmp + (uint64_t)l * (uint64_t)t.width,
                   (size_t)t.width);
    }
    free(tmp);
    free(b);
    return r;
}

/* ------------------------------------------------------------------ */
/* 7. Dequantization: w = bf16_rne(float(q - zero) * scale). */

static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb; /* round to nearest, ties to even (no NaN can reach here) */
    return (uint16_t)(u >> 16);
}

void or_dequant_bf16(const uint8_t *q, int64_t n, float scale, int32_t zero, uint16_t *out) {
    for (int64_t i = 0; i < n; i++) {
        float v = (float)((int32_t)q[i] - zero) * scale;
        out[i] = f32_to_bf16_rne(v);
    }
}

/* ------------------------------------------------------------------ */
/* 8. GEMV in double: y[b][r] = sum_k w[r][k] * x[b][k] over bf16 inputs. */

static double bf16_to_double(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

void or_gemv(const uint16_t *w, int64_t rows, int64_t cols, const uint16_t *x, int batch,
             int64_t r0, int64_t r1, double *y /* [batch][r1-r0] */, double *abs_sum) {
    (void)rows; /* w holds rows [r0, r1) only */
    for (int b = 0; b < batch; b++) {
        for (int64_t r = r0; r < r1; r++) {
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < cols; k++) {
                double t = bf16_to_double(w[(r - r0) * cols + k]) * bf16_to_double(x[(int64_t)b * cols + k]);
                acc += t;
                mag += fabs(t);
            }
            y[(int64_t)b * (r1 - r0) + (r - r0)] = acc;
            if (abs_sum) abs_sum[(int64_t)b * (r1 - r0) + (r - r0)] = mag;
        }
    }
}
