// encoder.cpp -- host side of libentro: tensor-level quantization, length-
// limited canonical Huffman codes and the chunked encoder, plus blob parsing.
//
// EntroLLM (arXiv 2505.02380v4), abstract and method details: per tensor,
// unsigned or asymmetric quantization chosen from the weight distribution;
// Huffman coding of the integer codes from their frequencies; the coded
// stream is cut into chunks that decode independently.  Code lengths are
// limited with package-merge (Larmore & Hirschberg, J. ACM 1990) and
// assigned canonically (RFC 1951 section 3.2.2) so the device decodes from
// length tables.  Everything here is deterministic and independent of the
// thread count.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <new>
#include <thread>
#include <vector>

#include "blob_format.h"
#include "entro.h"
#include "entro_internal.h"

namespace entro {

// ------------------------------------------------------------ threads

static int pick_threads(int requested, int64_t work) {
    int hw = (int)std::thread::hardware_concurrency();
    if (hw <= 0) hw = 1;
    int t = requested > 0 ? requested : hw;
    int64_t by_work = std::max<int64_t>(1, work / (int64_t(1) << 16));
    return (int)std::max<int64_t>(1, std::min<int64_t>(t, by_work));
}

template <class F>
static void parallel_for(int threads, int64_t count, F &&fn) {
    if (threads <= 1 || count <= 1) {
        if (count > 0) fn(0, count, 0);
        return;
    }
    threads = (int)std::min<int64_t>(threads, count);
    std::vector<std::thread> pool;
    pool.reserve(threads);
    for (int t = 0; t < threads; t++) {
        int64_t a = count * t / threads, b = count * (t + 1) / threads;
        pool.emplace_back([&fn, a, b, t] { fn(a, b, t); });
    }
    for (auto &th : pool) th.join();
}

// ------------------------------------------------------------ quantization

struct QuantParams {
    int scheme;
    float scale;
    int32_t zero;
    bool constant;
    uint8_t constant_code;
};

static inline uint8_t quant_one(float w, double scale, double zero, double qmax) {
    double v = std::nearbyint((double)w / scale) + zero;
    if (v < 0.0) v = 0.0;
    if (v > qmax) v = qmax;
    return (uint8_t)v;
}

static double entropy_bits(const int64_t *hist, int nsym) {
    int64_t n = 0;
    for (int i = 0; i < nsym; i++) n += hist[i];
    if (n == 0) return 0.0;
    double h = 0.0;
    for (int i = 0; i < nsym; i++)
        if (hist[i] > 0) {
            double p = (double)hist[i] / (double)n;
            h -= p * std::log2(p);
        }
    return h;
}

// Decide the scheme and its parameters; writes nothing to q.
static int choose_quant(const float *w, int64_t n, int bits, int mode, int threads, QuantParams *qp) {
    const int qmax = (1 << bits) - 1;
    qp->scheme = (mode == ENTRO_QUANT_ASYM) ? ENTRO_SCHEME_ASYM : ENTRO_SCHEME_UNSIGNED;
    qp->scale = 1.0f;
    qp->zero = 0;
    qp->constant = false;
    qp->constant_code = 0;
    if (n == 0) return ENTRO_OK;

    // min / max / finiteness
    std::vector<float> mins(threads, 0.f), maxs(threads, 0.f);
    std::vector<int> bad(threads, 0);
    parallel_for(threads, n, [&](int64_t a, int64_t b, int t) {
        float lo = w[a], hi = w[a];
        int nf = 0;
        for (int64_t i = a; i < b; i++) {
            float v = w[i];
            if (!std::isfinite(v)) nf = 1;
            lo = v < lo ? v : lo;
            hi = v > hi ? v : hi;
        }
        mins[t] = lo;
        maxs[t] = hi;
        bad[t] = nf;
    });
    float mn = w[0], mx = w[0];
    int used = (int)std::min<int64_t>(threads, n);
    for (int t = 0; t < used; t++) {
        if (bad[t]) return ENTRO_E_INVAL;
        mn = std::min(mn, mins[t]);
        mx = std::max(mx, maxs[t]);
    }
    if (mode == ENTRO_QUANT_UNSIGNED && mn < 0.0f) return ENTRO_E_INVAL;

    if (mx == mn) {
        if (mode == ENTRO_QUANT_AUTO) qp->scheme = (mn >= 0.0f) ? ENTRO_SCHEME_UNSIGNED : ENTRO_SCHEME_ASYM;
        qp->constant = true;
        qp->constant_code = (mn == 0.0f) ? 0 : 1;
        qp->scale = (mn == 0.0f) ? 1.0f : mn;
        return ENTRO_OK;
    }

    // candidates
    bool u_ok = false, a_ok = false;
    float su = 0.f, sa = 0.f;
    double za = 0.0;
    if (mode != ENTRO_QUANT_ASYM && mn >= 0.0f) {
        su = (float)((double)mx / (double)qmax);
        u_ok = (su > 0.0f) && !std::isinf(su);
    }
    if (mode != ENTRO_QUANT_UNSIGNED) {
        sa = (float)(((double)mx - (double)mn) / (double)qmax);
        if ((sa > 0.0f) && !std::isinf(sa)) {
            za = std::nearbyint(-(double)mn / (double)sa);
            a_ok = std::fabs(za) <= kMaxZero;
        }
    }
    if (mode == ENTRO_QUANT_UNSIGNED) {
        if (!u_ok) return ENTRO_E_LIMIT;
        qp->scheme = ENTRO_SCHEME_UNSIGNED;
        qp->scale = su;
        return ENTRO_OK;
    }
    if (mode == ENTRO_QUANT_ASYM) {
        if (!a_ok) return ENTRO_E_LIMIT;
        qp->scheme = ENTRO_SCHEME_ASYM;
        qp->scale = sa;
        qp->zero = (int32_t)za;
        return ENTRO_OK;
    }
    if (!u_ok && !a_ok) return ENTRO_E_LIMIT;
    bool take_unsigned;
    if (!a_ok) {
        take_unsigned = true;
    } else if (!u_ok) {
        take_unsigned = false;
    } else {
        // histograms of both candidates in one pass
        std::vector<int64_t> hu((size_t)threads * 256, 0), ha((size_t)threads * 256, 0);
        parallel_for(threads, n, [&](int64_t a, int64_t b, int t) {
            int64_t *lu = &hu[(size_t)t * 256], *la = &ha[(size_t)t * 256];
            for (int64_t i = a; i < b; i++) {
                lu[quant_one(w[i], (double)su, 0.0, qmax)]++;
                la[quant_one(w[i], (double)sa, za, qmax)]++;
            }
        });
        int64_t tu[256] = {0}, ta[256] = {0};
        for (int t = 0; t < threads; t++)
            for (int s = 0; s < 256; s++) {
                tu[s] += hu[(size_t)t * 256 + s];
                ta[s] += ha[(size_t)t * 256 + s];
            }
        double eu = entropy_bits(tu, qmax + 1), ea = entropy_bits(ta, qmax + 1);
        take_unsigned = eu <= ea + 1e-9;
    }
    if (take_unsigned) {
        qp->scheme = ENTRO_SCHEME_UNSIGNED;
        qp->scale = su;
        qp->zero = 0;
    } else {
        qp->scheme = ENTRO_SCHEME_ASYM;
        qp->scale = sa;
        qp->zero = (int32_t)za;
    }
    return ENTRO_OK;
}

static void apply_quant(const float *w, int64_t n, int bits, const QuantParams &qp, int threads, uint8_t *q) {
    const double qmax = (double)((1 << bits) - 1);
    parallel_for(threads, n, [&](int64_t a, int64_t b, int) {
        if (qp.constant) {
            std::memset(q + a, qp.constant_code, (size_t)(b - a));
            return;
        }
        const double s = (double)qp.scale, z = (double)qp.zero;
        for (int64_t i = a; i < b; i++) q[i] = quant_one(w[i], s, z, qmax);
    });
}

// ------------------------------------------------------------ code lengths
//
// Package-merge over lists that keep only weights and a leaf flag.  List d is
// merge(leaves, packages of list d+1), a leaf ahead of a package of equal
// weight; leaves are ordered by (count, symbol).  Selecting the 2m-2 lightest
// items at the top list and walking down, the selected prefix of list d+1 is
// twice the number of packages in the selected prefix of list d; a leaf of
// rank r gains one bit of length for every list whose selected prefix holds
// more than r leaves.

int code_lengths(const int64_t *hist, int nsym, int max_len, uint8_t *len) {
    if (nsym < 1 || nsym > 256 || max_len < 1 || max_len > kMaxLenLimit) return ENTRO_E_INVAL;
    std::vector<int> order;
    for (int s = 0; s < nsym; s++) {
        len[s] = 0;
        if (hist[s] < 0) return ENTRO_E_INVAL;
        if (hist[s] > 0) order.push_back(s);
    }
    const int m = (int)order.size();
    if (m == 0) return ENTRO_OK;
    if (m == 1) {
        len[order[0]] = 1;
        return ENTRO_OK;
    }
    if ((int64_t)m > (int64_t(1) << max_len)) return ENTRO_E_LIMIT;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return hist[a] < hist[b]; });
    std::vector<int64_t> leafw(m);
    for (int i = 0; i < m; i++) leafw[i] = hist[order[i]];

    // lists[d] for d = max_len (leaves only) down to 1; store weight + is_leaf.
    std::vector<std::vector<int64_t>> wts(max_len + 1);
    std::vector<std::vector<uint8_t>> leaf(max_len + 1);
    wts[max_len] = leafw;
    leaf[max_len].assign(m, 1);
    for (int d = max_len - 1; d >= 1; d--) {
        const std::vector<int64_t> &prev = wts[d + 1];
        const int np = (int)prev.size() / 2;
        std::vector<int64_t> &out = wts[d];
        std::vector<uint8_t> &fl = leaf[d];
        out.clear();
        fl.clear();
        out.reserve(m + np);
        fl.reserve(m + np);
        int li = 0, pi = 0;
        while (li < m || pi < np) {
            int64_t pw = pi < np ? prev[2 * pi] + prev[2 * pi + 1] : 0;
            if (pi >= np || (li < m && leafw[li] <= pw)) {
                out.push_back(leafw[li++]);
                fl.push_back(1);
            } else {
                out.push_back(pw);
                fl.push_back(0);
                pi++;
            }
        }
    }
    std::vector<int> depth_count(m, 0);
    int64_t take = 2 * (int64_t)m - 2;
    for (int d = 1; d <= max_len && take > 0; d++) {
        if (take > (int64_t)wts[d].size()) return ENTRO_E_LIMIT;
        int leaves = 0, packages = 0;
        for (int64_t i = 0; i < take; i++) {
            if (leaf[d][i]) leaves++;
            else packages++;
        }
        for (int r = 0; r < leaves; r++) depth_count[r]++;
        take = 2 * (int64_t)packages;
    }
    for (int r = 0; r < m; r++) len[order[r]] = (uint8_t)depth_count[r];
    return ENTRO_OK;
}

void canonical_codes(const uint8_t *len, uint32_t *code) {
    int count[kMaxLenLimit + 2] = {0};
    for (int s = 0; s < 256; s++)
        if (len[s]) count[len[s]]++;
    uint32_t next[kMaxLenLimit + 2] = {0};
    uint32_t c = 0;
    for (int l = 1; l <= kMaxLenLimit; l++) {
        c = (c + (uint32_t)count[l - 1]) << 1;
        next[l] = c;
    }
    for (int s = 0; s < 256; s++) code[s] = len[s] ? next[len[s]]++ : 0;
}

// ------------------------------------------------------------ bit writer

struct BitSink {
    uint32_t *dst;     // word pointer (lanes: strided by 32)
    int64_t stride;    // word stride
    uint64_t acc = 0;  // pending bits, MSB-aligned
    int nacc = 0;
    int64_t widx = 0;
    void put(uint32_t code, int l) {
        acc |= (uint64_t)code << (64 - nacc - l);
        nacc += l;
        if (nacc >= 32) {
            dst[widx * stride] = (uint32_t)(acc >> 32);
            widx++;
            acc <<= 32;
            nacc -= 32;
        }
    }
    void flush() {
        if (nacc > 0) {
            dst[widx * stride] = (uint32_t)(acc >> 32);
            widx++;
            acc = 0;
            nacc = 0;
        }
    }
};

// ------------------------------------------------------------ encoder

// One tile in consumption order (the layout is described in blob_format.h).
// Each lane's words are coded on their own; a pass over each lane's code
// lengths finds the refill points where it takes its later words; sorting the
// takes by (refill point, lane) gives their places.
static int write_consumption_tile(const TileGeom &t, const uint8_t *q, int64_t cols, int L, int bits, int max_len,
                                  int count_bytes, const uint32_t *code, const uint8_t *len, uint32_t *dst,
                                  uint64_t dst_words) {
    const int per_lookup = bits == 4 ? kCoCodes4 : kCoCodes8;
    const bool each = max_len > kCoRefillEachAbove;
    std::vector<std::vector<uint32_t>> words((size_t)L);
    struct Take {
        uint64_t point;
        int lane;
        uint32_t word;
    };
    std::vector<Take> takes;
    std::vector<uint8_t> lens((size_t)t.width);
    for (int l = 0; l < t.nrows; l++) {
        const uint8_t *row = q + (t.row0 + l) * cols + t.col0;
        uint64_t bits_l = 0;
        for (int64_t k = 0; k < t.width; k++) {
            lens[(size_t)k] = len[row[k]];
            bits_l += len[row[k]];
        }
        std::vector<uint32_t> &w = words[(size_t)l];
        w.assign((size_t)((bits_l + 31) / 32) + 1, 0u);
        BitSink s{w.data(), 1};
        for (int64_t k = 0; k < t.width; k++) s.put(code[row[k]], len[row[k]]);
        s.flush();
        w.resize((size_t)((bits_l + 31) / 32));
        // the lane's refill points: count the bits each lookup takes
        size_t next_word = std::min<size_t>(3, w.size());
        int64_t i = 0;
        uint32_t used_since = 0;
        for (uint64_t j = 0; next_word < w.size(); j++) {
            if ((each || (j & 1) == 0) && used_since >= 32) {
                used_since -= 32;
                takes.push_back({each ? j : j / 2, l, w[next_word++]});
                if (next_word == w.size()) break;
            }
            if (i >= t.width) return ENTRO_E_INVAL;  // cannot happen: words left means codes left
            if (lens[(size_t)i] > kCoPeekBits) {
                used_since += lens[(size_t)i++];
                continue;
            }
            uint32_t peek = 0;
            for (int k = 0; k < per_lookup && i < t.width && peek + lens[(size_t)i] <= (uint32_t)kCoPeekBits; k++)
                peek += lens[(size_t)i++];
            used_since += peek;
        }
    }
    std::stable_sort(takes.begin(), takes.end(), [](const Take &a, const Take &b) {
        return a.point != b.point ? a.point < b.point : a.lane < b.lane;
    });
    const uint64_t hw = co_header_words((uint64_t)L, count_bytes);
    const uint64_t need = hw + 3 * (uint64_t)L + takes.size();
    if (((need + 3) & ~3ull) != dst_words) return ENTRO_E_INVAL;
    std::memset(dst, 0, dst_words * 4);
    uint8_t *hdr = reinterpret_cast<uint8_t *>(dst);  // little-endian host
    for (int l = 0; l < L; l++) {
        const uint32_t nw = (uint32_t)words[(size_t)l].size();
        hdr[count_bytes * l] = (uint8_t)nw;
        if (count_bytes == 2) hdr[2 * l + 1] = (uint8_t)(nw >> 8);
    }
    for (int r = 0; r < 3; r++)
        for (int l = 0; l < L; l++)
            if ((size_t)r < words[(size_t)l].size()) dst[hw + (uint64_t)L * r + l] = words[(size_t)l][(size_t)r];
    uint64_t p = hw + 3 * (uint64_t)L;
    for (const Take &tk : takes) dst[p++] = tk.word;
    return ENTRO_OK;
}

static int encode_impl(const float *w, int64_t rows, int64_t cols, const entro_encode_opts *o, Blob **out) {
    if (!out || !o || rows < 0 || cols < 0) return ENTRO_E_INVAL;
    if ((rows * cols > 0) && !w) return ENTRO_E_INVAL;
    if (o->bits != 4 && o->bits != 8) return ENTRO_E_INVAL;
    if (o->quant_mode < 0 || o->quant_mode > 2) return ENTRO_E_INVAL;
    if (o->format != ENTRO_FORMAT_SINGLE && o->format != ENTRO_FORMAT_LANES && o->format != ENTRO_FORMAT_ROWS &&
        o->format != ENTRO_FORMAT_ROWS_CO)
        return ENTRO_E_INVAL;
    if (o->threads < 0) return ENTRO_E_INVAL;
    const int bits = o->bits, nsym = 1 << bits;
    const int max_len = o->max_len ? o->max_len : (bits == 8 ? 16 : 12);
    if (max_len < 1 || max_len > kMaxLenLimit) return ENTRO_E_INVAL;
    const bool consume = o->format == ENTRO_FORMAT_ROWS_CO;
    const bool tiles = o->format == ENTRO_FORMAT_ROWS || consume;
    const bool lanes = o->format == ENTRO_FORMAT_LANES || tiles;  // lane bitstreams
    const int L = lanes ? (o->lanes ? o->lanes : kLanes) : 1;
    if (lanes && L != 32 && L != 64) return ENTRO_E_INVAL;
    const int64_t step = (int64_t)kRun * L;
    int64_t C = o->chunk_symbols ? o->chunk_symbols : (lanes ? 8192 : 4096);
    if (lanes && (C < step || C > kMaxLanesChunk || C % step)) return ENTRO_E_INVAL;
    if (!lanes && (C < 1 || C > kMaxSingleChunk)) return ENTRO_E_INVAL;
    if (tiles && cols % kRun) return ENTRO_E_INVAL;
    const int64_t n = rows * cols;
    const int threads = pick_threads(o->threads, n);

    QuantParams qp;
    int r = choose_quant(w, n, bits, o->quant_mode, threads, &qp);
    if (r != ENTRO_OK) return r;
    std::vector<uint8_t> q;
    try {
        q.resize((size_t)std::max<int64_t>(n, 1));
    } catch (const std::bad_alloc &) {
        return ENTRO_E_NOMEM;
    }
    apply_quant(w, n, bits, qp, threads, q.data());

    // histogram
    std::vector<int64_t> th((size_t)threads * 256, 0);
    parallel_for(threads, n, [&](int64_t a, int64_t b, int t) {
        int64_t *h = &th[(size_t)t * 256];
        for (int64_t i = a; i < b; i++) h[q[i]]++;
    });
    int64_t hist[256] = {0};
    for (int t = 0; t < threads; t++)
        for (int s = 0; s < 256; s++) hist[s] += th[(size_t)t * 256 + s];

    uint8_t len[256] = {0};
    r = code_lengths(hist, nsym, max_len, len);
    if (r != ENTRO_OK) return r;
    uint32_t code[256];
    canonical_codes(len, code);

    const uint64_t n_chunks = tiles ? tile_count((uint64_t)rows, (uint64_t)cols, (uint64_t)L, (uint64_t)C)
                                    : n > 0 ? (uint64_t)((n + C - 1) / C) : 0;
    std::vector<uint64_t> start(n_chunks + 1, 0);
    const int count_bytes = co_count_bytes((uint64_t)(C / L), (uint32_t)max_len);

    // pass 1: per-chunk size (bits for single stream, words for lanes)
    std::vector<uint64_t> csize(n_chunks, 0);
    parallel_for(threads, (int64_t)n_chunks, [&](int64_t c0, int64_t c1, int) {
        for (int64_t c = c0; c < c1; c++) {
            const int64_t a = c * C, b = std::min<int64_t>(n, a + C);
            if (tiles) {
                const TileGeom t = tile_geom((uint64_t)rows, (uint64_t)cols, (uint64_t)L, (uint64_t)C, (uint64_t)c);
                uint64_t wmax = 0, later = 0;
                for (int l = 0; l < t.nrows; l++) {
                    const uint8_t *row = q.data() + (t.row0 + l) * cols + t.col0;
                    uint64_t s = 0;
                    for (int64_t k = 0; k < t.width; k++) s += len[row[k]];
                    wmax = std::max<uint64_t>(wmax, (s + 31) / 32);
                    later += (s + 31) / 32 > 3 ? (s + 31) / 32 - 3 : 0;
                }
                csize[c] = consume ? (co_header_words((uint64_t)L, count_bytes) + 3 * (uint64_t)L + later + 3) & ~3ull
                                   : wmax * (uint64_t)L;
            } else if (!lanes) {
                uint64_t s = 0;
                for (int64_t i = a; i < b; i++) s += len[q[i]];
                csize[c] = s;
            } else {
                uint64_t lb[kMaxLanes] = {0};
                for (int64_t p = 0; p < b - a; p++) lb[(p % step) / kRun] += len[q[a + p]];
                uint64_t wmax = 0;
                for (int l = 0; l < L; l++) wmax = std::max<uint64_t>(wmax, (lb[l] + 31) / 32);
                csize[c] = wmax * (uint64_t)L;
            }
        }
    });
    for (uint64_t c = 0; c < n_chunks; c++) start[c + 1] = start[c] + csize[c];
    const uint64_t payload_words = lanes ? start[n_chunks] : (start[n_chunks] + 31) / 32;

    Blob *blob = new (std::nothrow) Blob();
    if (!blob) return ENTRO_E_NOMEM;
    const uint64_t total = payload_offset(n_chunks) + 4 * payload_words;
    try {
        blob->bytes.assign((size_t)total, 0);
    } catch (const std::bad_alloc &) {
        delete blob;
        return ENTRO_E_NOMEM;
    }
    uint8_t *base = blob->bytes.data();
    BlobHeader h;
    std::memset(&h, 0, sizeof(h));
    h.magic = kMagic;
    h.version = kVersion;
    h.bits = (uint32_t)bits;
    h.scheme = (uint32_t)qp.scheme;
    h.max_len = (uint32_t)max_len;
    h.format = (uint32_t)o->format;
    h.lanes = (uint32_t)L;
    h.run = lanes ? kRun : 1;
    h.rows = (uint64_t)rows;
    h.cols = (uint64_t)cols;
    h.n = (uint64_t)n;
    h.chunk_symbols = (uint64_t)C;
    h.n_chunks = n_chunks;
    std::memcpy(&h.scale_bits, &qp.scale, 4);
    h.zero = qp.zero;
    h.payload_words = payload_words;
    std::memcpy(base, &h, sizeof(h));  // the host is little-endian (x86-64 / aarch64)
    std::memcpy(base + kHeaderBytes, len, 256);
    uint64_t *idx = reinterpret_cast<uint64_t *>(base + index_offset());
    for (uint64_t c = 0; c <= n_chunks; c++) {
        idx[2 * c] = start[c];
        idx[2 * c + 1] = std::min<uint64_t>((uint64_t)n, c * (uint64_t)C);
        if (tiles)
            idx[2 * c + 1] = c < n_chunks ? tile_geom((uint64_t)rows, (uint64_t)cols, (uint64_t)L, (uint64_t)C, c).first
                                          : (uint64_t)n;
    }
    uint32_t *payload = reinterpret_cast<uint32_t *>(base + payload_offset(n_chunks));

    // pass 2: bits
    std::atomic<int> failed{ENTRO_OK};
    parallel_for(threads, (int64_t)n_chunks, [&](int64_t c0, int64_t c1, int) {
        std::vector<uint32_t> tmp;
        for (int64_t c = c0; c < c1; c++) {
            const int64_t a = c * C, b = std::min<int64_t>(n, a + C);
            if (consume) {
                const TileGeom t = tile_geom((uint64_t)rows, (uint64_t)cols, (uint64_t)L, (uint64_t)C, (uint64_t)c);
                const int r2 = write_consumption_tile(t, q.data(), cols, L, bits, max_len, count_bytes, code, len,
                                                      payload + start[c], start[c + 1] - start[c]);
                if (r2 != ENTRO_OK) failed.store(r2, std::memory_order_relaxed);
            } else if (tiles) {
                const TileGeom t = tile_geom((uint64_t)rows, (uint64_t)cols, (uint64_t)L, (uint64_t)C, (uint64_t)c);
                uint32_t *cbase = payload + start[c];
                for (int l = 0; l < t.nrows; l++) {
                    BitSink s{cbase + l, L};
                    const uint8_t *row = q.data() + (t.row0 + l) * cols + t.col0;
                    for (int64_t k = 0; k < t.width; k++) s.put(code[row[k]], len[row[k]]);
                    s.flush();
                }
            } else if (!lanes) {
                // chunks are bit-contiguous: write this chunk's bits into a
                // private word buffer aligned like the payload, then OR the
                // edge words (shared with neighbours) atomically.
                const uint64_t bit0 = start[c], bit1 = start[c + 1];
                if (bit1 == bit0) continue;
                const uint64_t w0 = bit0 / 32, w1 = (bit1 + 31) / 32;
                tmp.assign(w1 - w0, 0);
                BitSink s{tmp.data(), 1};
                s.acc = 0;
                s.nacc = (int)(bit0 % 32);  // leading bits belong to the previous chunk
                for (int64_t i = a; i < b; i++) s.put(code[q[i]], len[q[i]]);
                s.flush();
                for (uint64_t j = 0; j < w1 - w0; j++) {
                    const bool edge = (j == 0) || (j + 1 == w1 - w0);
                    if (edge) __atomic_fetch_or(&payload[w0 + j], tmp[j], __ATOMIC_RELAXED);
                    else payload[w0 + j] = tmp[j];
                }
            } else {
                uint32_t *cbase = payload + start[c];
                for (int l = 0; l < L; l++) {
                    BitSink s{cbase + l, L};
                    for (int64_t t0 = 0; t0 < b - a; t0 += step) {
                        const int64_t p0 = t0 + (int64_t)l * kRun;
                        const int64_t p1 = std::min<int64_t>(b - a, p0 + kRun);
                        for (int64_t p = p0; p < p1; p++) s.put(code[q[a + p]], len[q[a + p]]);
                    }
                    s.flush();
                }
            }
        }
    });
    r = failed.load();
    if (r == ENTRO_OK) r = blob->finalize_info();
    if (r != ENTRO_OK) {
        delete blob;
        return r;
    }
    uint64_t cb = 0;
    for (int s = 0; s < 256; s++) cb += (uint64_t)hist[s] * len[s];
    blob->coded_bits = cb;
    *out = blob;
    return ENTRO_OK;
}

// ------------------------------------------------------------ parsing

int Blob::finalize_info() {
    const uint8_t *base = bytes.data();
    if (bytes.size() < (size_t)index_offset()) return ENTRO_E_FORMAT;
    std::memcpy(&header, base, sizeof(header));
    std::memcpy(lengths, base + kHeaderBytes, 256);
    const BlobHeader &h = header;
    if (h.magic != kMagic || h.version != kVersion) return ENTRO_E_FORMAT;
    if (h.bits != 4 && h.bits != 8) return ENTRO_E_FORMAT;
    if (h.scheme > 1) return ENTRO_E_FORMAT;
    if (h.max_len < 1 || h.max_len > (uint32_t)kMaxLenLimit) return ENTRO_E_FORMAT;
    const bool consume = h.format == ENTRO_FORMAT_ROWS_CO;
    const bool tiles = h.format == ENTRO_FORMAT_ROWS || consume;
    const bool lanes = h.format == ENTRO_FORMAT_LANES || tiles;
    if (!lanes && h.format != ENTRO_FORMAT_SINGLE) return ENTRO_E_FORMAT;
    if (lanes ? (h.lanes != 32 && h.lanes != 64) : h.lanes != 1) return ENTRO_E_FORMAT;
    if (h.run != (lanes ? (uint32_t)kRun : 1u)) return ENTRO_E_FORMAT;
    if (h.chunk_symbols == 0) return ENTRO_E_FORMAT;
    if (lanes && (h.chunk_symbols % (kRun * h.lanes) || h.chunk_symbols > (uint64_t)kMaxLanesChunk))
        return ENTRO_E_FORMAT;
    if (!lanes && h.chunk_symbols > (uint64_t)kMaxSingleChunk) return ENTRO_E_FORMAT;
    if (h.cols != 0 && h.rows > UINT64_MAX / h.cols) return ENTRO_E_FORMAT;
    if (h.n != h.rows * h.cols) return ENTRO_E_FORMAT;
    if (tiles && h.cols % kRun) return ENTRO_E_FORMAT;
    if (h.n_chunks != (tiles ? tile_count(h.rows, h.cols, h.lanes, h.chunk_symbols)
                             : (h.n + h.chunk_symbols - 1) / h.chunk_symbols))
        return ENTRO_E_FORMAT;
    if (h.n_chunks > (uint64_t(1) << 40) || h.payload_words > (uint64_t(1) << 40)) return ENTRO_E_FORMAT;
    if (bytes.size() != (size_t)(payload_offset(h.n_chunks) + 4 * h.payload_words)) return ENTRO_E_FORMAT;
    int nz = 0;
    for (int s = 0; s < 256; s++) {
        if (lengths[s] > h.max_len) return ENTRO_E_FORMAT;
        if (lengths[s] && s >= (1 << h.bits)) return ENTRO_E_FORMAT;
        nz += lengths[s] != 0;
    }
    if (h.n > 0 && nz == 0) return ENTRO_E_FORMAT;
    // Kraft: a complete code, or one symbol of length 1
    if (nz >= 2) {
        uint64_t k = 0;
        for (int s = 0; s < 256; s++)
            if (lengths[s]) k += uint64_t(1) << (h.max_len - lengths[s]);
        if (k != (uint64_t(1) << h.max_len)) return ENTRO_E_FORMAT;
    } else if (nz == 1) {
        for (int s = 0; s < 256; s++)
            if (lengths[s] && lengths[s] != 1) return ENTRO_E_FORMAT;
    }
    const uint64_t *idx = reinterpret_cast<const uint64_t *>(base + index_offset());
    uint64_t maxw = 0, prev = 0;
    for (uint64_t c = 0; c <= h.n_chunks; c++) {
        const uint64_t st = idx[2 * c], first = idx[2 * c + 1];
        const uint64_t want = !tiles ? std::min<uint64_t>(h.n, c * h.chunk_symbols)
                              : c < h.n_chunks ? tile_geom(h.rows, h.cols, h.lanes, h.chunk_symbols, c).first
                                               : h.n;
        if (first != want) return ENTRO_E_FORMAT;
        if (c == 0 ? st != 0 : st < prev) return ENTRO_E_FORMAT;
        if (c > 0 && lanes) {
            const uint64_t wc = st - prev;
            if (consume) {  // header + three rows at least, whole 16-byte groups
                if (wc % 4 || wc < co_header_words(h.lanes, co_count_bytes(h.chunk_symbols / h.lanes, h.max_len)) +
                                       3ull * h.lanes)
                    return ENTRO_E_FORMAT;
                maxw = std::max<uint64_t>(maxw, (wc + h.lanes - 1) / h.lanes);
            } else {
                if (wc % h.lanes) return ENTRO_E_FORMAT;
                maxw = std::max<uint64_t>(maxw, wc / h.lanes);
            }
        }
        if (c > 0 && !lanes) maxw = std::max<uint64_t>(maxw, (st + 31) / 32 - prev / 32);
        prev = st;
    }
    if (lanes ? prev != h.payload_words : (prev + 31) / 32 != h.payload_words) return ENTRO_E_FORMAT;
    max_chunk_words = maxw;
    coded_bits = lanes ? 0 : prev;  // lanes: known only to the encoder (padding is not code)
    return ENTRO_OK;
}

}  // namespace entro

using entro::Blob;

extern "C" int entro_encode(const float *host_w, int64_t rows, int64_t cols, const entro_encode_opts *opts,
                            entro_blob **out) {
    if (!out) return ENTRO_E_INVAL;
    *out = nullptr;
    Blob *b = nullptr;
    int r = entro::encode_impl(host_w, rows, cols, opts, &b);
    if (r == ENTRO_OK) *out = reinterpret_cast<entro_blob *>(b);
    return r;
}

extern "C" int entro_blob_from_bytes(const void *data, uint64_t size, entro_blob **out) {
    if (!out || (!data && size)) return ENTRO_E_INVAL;
    *out = nullptr;
    Blob *b = new (std::nothrow) Blob();
    if (!b) return ENTRO_E_NOMEM;
    try {
        b->bytes.assign((const uint8_t *)data, (const uint8_t *)data + size);
    } catch (const std::bad_alloc &) {
        delete b;
        return ENTRO_E_NOMEM;
    }
    int r = b->finalize_info();
    if (r != ENTRO_OK) {
        delete b;
        return r;
    }
    *out = reinterpret_cast<entro_blob *>(b);
    return ENTRO_OK;
}

extern "C" int entro_blob_bytes(const entro_blob *blob, const void **data, uint64_t *size) {
    if (!blob || !data || !size) return ENTRO_E_INVAL;
    const Blob *b = reinterpret_cast<const Blob *>(blob);
    *data = b->bytes.data();
    *size = b->bytes.size();
    return ENTRO_OK;
}

extern "C" int entro_blob_info(const entro_blob *blob, entro_info *out) {
    if (!blob || !out) return ENTRO_E_INVAL;
    const Blob *b = reinterpret_cast<const Blob *>(blob);
    const entro::BlobHeader &h = b->header;
    std::memset(out, 0, sizeof(*out));
    out->bits = (int32_t)h.bits;
    out->scheme = (int32_t)h.scheme;
    out->max_len = (int32_t)h.max_len;
    out->format = (int32_t)h.format;
    out->rows = (int64_t)h.rows;
    out->cols = (int64_t)h.cols;
    out->n = (int64_t)h.n;
    out->chunk_symbols = (int64_t)h.chunk_symbols;
    out->n_chunks = (int64_t)h.n_chunks;
    std::memcpy(&out->scale, &h.scale_bits, 4);
    out->zero = h.zero;
    out->payload_bytes = 4 * h.payload_words;
    out->index_bytes = 16 * (h.n_chunks + 1);
    out->blob_bytes = b->bytes.size();
    out->max_chunk_words = (uint32_t)b->max_chunk_words;
    out->lanes = h.lanes;
    std::memcpy(out->lengths, b->lengths, 256);
    out->coded_bits = b->coded_bits;
    return ENTRO_OK;
}

extern "C" void entro_blob_free(entro_blob *blob) { delete reinterpret_cast<Blob *>(blob); }
