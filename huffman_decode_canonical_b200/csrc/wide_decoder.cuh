// wide_decoder.cuh -- the lane decoder with two-word table entries, shared by
// the lanes-format kernels (decode.cu) and the row-tile kernel (rows.cuh).
// Included by decode.cu inside namespace entro, after the shared helpers.
//
// Each lane keeps a 64-bit MSB-first window of its bitstream in two registers
// and peeks 12 bits into a table of two-word entries {codes, meta}: up to 8
// 4-bit or 4 8-bit whole codes of the peek (EntroLLM, arXiv 2505.02380v4: the
// Huffman-coded chunks decode in parallel; several codes per table lookup),
// and meta = bits they take | (codes * BITS) << 8.  A counter register C holds
// the window bits consumed (bits 0-7), the pending code bits (bits 8-15) and
// the runs completed (bits 16-31), so that adding meta to C does both counts
// at once and meta itself is the window's shift amount.  Codes longer than 12
// bits take the canonical slow path.  Every 8 codes form a run, stored in a
// slot of shared memory in output order.

constexpr uint32_t kPbShift = 8;             // pending code bits: bits 8-15 of the counter
constexpr uint32_t kRunsShift = 16;          // runs completed: bits 16-31 of the counter

__host__ __device__ constexpr int wide_max_codes(int bits) { return bits == 4 ? 8 : 4; }

// Runs a lane may complete past the check that stops it: STEPS lookups of at
// most wide_max_codes codes on top of at most 7 pending codes.
__host__ __device__ constexpr int wide_runs_per_check(int bits, int steps) {
    return (kRun - 1 + steps * wide_max_codes(bits)) / kRun;
}


__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

// Integer constants the compiler cannot see (kernel arguments: 1 and powers of
// two).  A shift or an addition written as a multiply-add with one of them
// runs on the FMA pipe (IMAD) instead of the ALU pipe, which the lookups would
// otherwise saturate: the decode and its emission split their integer work
// over both pipes.
struct Pipes {
    uint32_t one, four, eight, two8, two12, two24;
};

__device__ __forceinline__ uint32_t imad(uint32_t a, uint32_t b, uint32_t c) {  // a * b + c
    uint32_t d;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t imulhi(uint32_t a, uint32_t b) {  // (a * b) >> 32
    uint32_t d;
    asm("mul.hi.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t byte_of(uint32_t v, uint32_t sel) {  // byte sel of v, zero-extended
    return __byte_perm(v, 0u, 0x4440u | sel);
}

// RB: bytes from a lane's slot of run t to its slot of run t + 1.  RING = 0:
// every run has its own slot; RING > 0: RING slots used in turn (run t in slot
// t mod RING).  CO: the chunk's words are in consumption order (row tiles,
// format 4): after its first three words a lane takes its next word from a
// cursor shared by the warp, in lane order among the lanes that refill at the
// same point (a ballot and a population count), and only while it has words
// left; the loop that drives it must keep the warp converged.
template <int BITS, bool SLOW, int LANES, uint32_t RB, int RING, bool CO = false>
struct WideDecoder {
    static constexpr uint32_t kRowBytes = 4 * LANES;  // one staged word of every lane
    static constexpr uint32_t kRunBytes = RB;
    // Load the next lookup's entry before the append, so that the append's work
    // hides the load (8-bit codes, and the ring of the lanes kernel), or at the
    // lookup (4-bit row tiles: measured faster that way).
    static constexpr bool kAhead = BITS == 8 || RING > 0;
    uint32_t tab;         // shared address of the {codes, meta} table
    uint32_t bufa;        // shared address of the word held in wnext (a refill advances, then loads)
    uint32_t bufcap;      // shared address of this lane's last readable word
    uint32_t hi, lo;      // 64-bit window, MSB first
    uint32_t wnext;       // next word, loaded one refill ahead
    uint32_t C;           // consumed window bits | pending bits << 8 | runs << 16
    uint32_t p0, p1;      // pending codes as one bit string, first code at bit 0 of p0 (p1: 8-bit only)
    uint32_t osta;        // shared address of the current run's slot
    uint32_t rend;        // RING > 0: address one ring past this lane's slot of run 0
    uint32_t cur;         // CO: shared address of the chunk's next unplaced word (same in every lane)
    uint32_t left;        // CO: words this lane has still to take
    uint32_t lt;          // CO: the lanes below this one
    uint2 e;              // table entry of the window's top 12 bits, loaded one lookup ahead

    // b: shared address of this lane's word 0 (word j at b + kRowBytes j);
    // slot0: its slot of run 0; cap: last readable staging row.
    __device__ __forceinline__ void init(const Pipes &k, uint32_t table, uint32_t b, uint32_t slot0, int cap,
                                         bool active) {
        tab = table;
        bufcap = b + kRowBytes * static_cast<uint32_t>(cap);
        hi = lds32(b);
        lo = lds32(b + kRowBytes);
        bufa = b + 2 * kRowBytes;
        wnext = lds32(min(bufa, bufcap));
        C = active ? 0u : 0xFFFF0000u;  // an empty lane counts as done
        p0 = p1 = 0;
        osta = slot0;
        rend = slot0 + static_cast<uint32_t>(RING) * RB;
        e = entry(k);
    }

    // Consumption order: b = this lane's word 0 (rows of kRowBytes as above),
    // next = the chunk's first word after the three rows, words = the words this
    // lane has after those three, last = the chunk's last word.
    __device__ __forceinline__ void init_co(const Pipes &k, uint32_t table, uint32_t b, uint32_t slot0, uint32_t next,
                                           uint32_t words, uint32_t last, bool active) {
        tab = table;
        bufa = b;
        bufcap = last;
        hi = lds32(b);
        lo = lds32(b + kRowBytes);
        wnext = lds32(b + 2 * kRowBytes);
        C = active ? 0u : 0xFFFF0000u;
        p0 = p1 = 0;
        osta = slot0;
        rend = slot0 + static_cast<uint32_t>(RING) * RB;
        cur = next;
        left = words;
        asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt));
        e = entry(k);
    }

    __device__ __forceinline__ int runs() const { return static_cast<int>(C >> kRunsShift); }

    // When 32 or more window bits are consumed (the valid bits then all sit in
    // hi and lo is zero), the next word lands right below them.
    __device__ __forceinline__ void refill(const Pipes &k) {
        if (CO) {
            // every lane of the warp runs this (the ballot); a lane that refills and has words
            // left takes the word at cur + 4 * (refilling lanes below it)
            asm volatile(
                "{\n\t"
                ".reg .pred p, t;\n\t"
                ".reg .u32 x, m, r, a;\n\t"
                "and.b32 x, %2, 32;\n\t"
                "setp.ne.u32 p, x, 0;\n\t"
                "setp.ne.and.u32 t, %5, 0, p;\n\t"
                "vote.sync.ballot.b32 m, t, 0xffffffff;\n\t"
                "and.b32 r, m, %7;\n\t"
                "popc.b32 r, r;\n\t"
                "@p shf.l.wrap.b32 x, %3, 0, %2;\n\t"  // wnext >> (32 - s), s = consumed - 32
                "@p mad.lo.u32 %0, x, %8, %0;\n\t"     // hi |= x
                "@p shf.l.wrap.b32 %1, 0, %3, %2;\n\t"  // wnext << s
                "@p mad.lo.u32 %2, %8, %9, %2;\n\t"    // consumed - 32
                "@t mad.lo.u32 a, r, %10, %4;\n\t"
                "@t min.u32 a, a, %6;\n\t"
                "@t ld.shared.u32 %3, [a];\n\t"
                "@t sub.u32 %5, %5, 1;\n\t"
                "popc.b32 m, m;\n\t"
                "mad.lo.u32 %4, m, %10, %4;\n\t"
                "}"
                : "+r"(hi), "+r"(lo), "+r"(C), "+r"(wnext), "+r"(cur), "+r"(left)
                : "r"(bufcap), "r"(lt), "r"(k.one), "r"(0xFFFFFFE0u), "r"(k.four)
                : "memory");
            return;
        }
        asm volatile(
            "{\n\t"
            ".reg .pred p;\n\t"
            ".reg .u32 x, a;\n\t"
            "and.b32 x, %2, 32;\n\t"
            "setp.ne.u32 p, x, 0;\n\t"
            "@p shf.l.wrap.b32 x, %3, 0, %2;\n\t"  // wnext >> (32 - s), s = consumed - 32
            "@p mad.lo.u32 %0, x, %6, %0;\n\t"     // hi |= x (x lands on hi's zero bits)
            "@p shf.l.wrap.b32 %1, 0, %3, %2;\n\t"  // wnext << s
            "@p mad.lo.u32 %2, %6, %7, %2;\n\t"    // consumed - 32
            "@p mad.lo.u32 %4, %6, %8, %4;\n\t"    // next word
            "@p min.u32 a, %4, %5;\n\t"
            "@p ld.shared.u32 %3, [a];\n\t"
            "}"
            : "+r"(hi), "+r"(lo), "+r"(C), "+r"(wnext), "+r"(bufa)
            : "r"(bufcap), "r"(k.one), "r"(0xFFFFFFE0u), "r"(kRowBytes)
            : "memory");
    }

    __device__ __forceinline__ uint2 entry(const Pipes &k) const {
        return lds64(imad(imulhi(hi, k.two12), k.eight, tab));  // table[window >> 52]
    }

    // One lookup.  e, the entry of the window's top 12 bits, is loaded here or
    // (kAhead) was loaded by the lookup before (or by init); for a code longer
    // than 12 bits the canonical slow path gives the single code instead.  The
    // window moves past the codes, a refill follows when r (a refill point
    // comes next) and the codes are appended to the current run; with kAhead
    // the next entry's load is issued before the append, whose integer work
    // then runs while the load is in flight.  live = false (a lane at its
    // chunk's end, kept in step with its warp) makes the lookup a no-op.
    __device__ __forceinline__ void step(const Pipes &k, bool r, const uint32_t *slim, const int32_t *soffs,
                                         const uint8_t *ssyms, int max_len, int32_t *status, bool live = true) {
        if (!kAhead) e = entry(k);
        uint32_t codes = live ? e.x : 0u, meta = live ? e.y : 0u;
        if (SLOW && live && (meta & 31u) == 0) {
            const uint64_t win = (static_cast<uint64_t>(hi) << 32) | lo;
            const uint32_t se = slow_entry(win, max_len, slim, soffs, ssyms, status);
            codes = (se >> 8) & 0xFFu;
            meta = (se & 31u) | (static_cast<uint32_t>(BITS) << kPbShift);
        }
        const uint32_t q = shift(k, meta);
        if (kAhead) {
            if (r) refill(k);
            e = entry(k);
            append(k, codes, q);
        } else {
            append(k, codes, q);
            if (r) refill(k);
        }
    }

    // Move the window past meta's bits and add meta to C; returns the pending
    // bits before this lookup's codes (C >> 8; the shifts use it mod 32).
    __device__ __forceinline__ uint32_t shift(const Pipes &k, uint32_t meta) {
        uint32_t q;
        asm volatile(
            "mul.hi.u32 %0, %3, %5;\n\t"
            "shf.l.wrap.b32 %1, %2, %1, %4;\n\t"
            "shf.l.wrap.b32 %2, 0, %2, %4;\n\t"
            "mad.lo.u32 %3, %4, %6, %3;\n\t"  // C += meta
            : "=r"(q), "+r"(hi), "+r"(lo), "+r"(C)
            : "r"(meta), "r"(k.two24), "r"(k.one));
        return q;
    }

    // Append the codes to the pending string at bit q, store the run's slot,
    // and move to the next slot when a run is whole.  Appends land on zero bits
    // of the string, so they are additions.
    __device__ __forceinline__ void append(const Pipes &k, uint32_t codes, uint32_t q) {
        if (BITS == 4 && RING == 0) {
            // every run of a slot-per-run buffer completes (row tiles: Kc is a multiple of 8),
            // so a lane stores its run word once, when the run is whole; what passes bit 32
            // (phi) starts the next run (pending bits < 32 before the append)
            asm volatile(
                "{\n\t"
                ".reg .u32 plo, phi, x;\n\t"
                ".reg .pred dn;\n\t"
                "shf.l.wrap.b32 plo, 0, %4, %5;\n\t"
                "shf.l.wrap.b32 phi, %4, 0, %5;\n\t"
                "mad.lo.u32 %0, plo, %6, %0;\n\t"
                "and.b32 x, %1, 0x2000;\n\t"
                "setp.ne.u32 dn, x, 0;\n\t"
                "@dn st.shared.u32 [%2], %0;\n\t"
                "selp.b32 %0, phi, %0, dn;\n\t"
                "@dn mad.lo.u32 %1, %6, %7, %1;\n\t"  // runs + 1, pending - 32
                "@dn mad.lo.u32 %2, %6, %3, %2;\n\t"
                "}"
                : "+r"(p0), "+r"(C), "+r"(osta)
                : "r"(kRunBytes), "r"(codes), "r"(q), "r"(k.one), "r"(0xE000u)
                : "memory");
        } else if (BITS == 4) {
            // a ring: the slot holds the run so far after every lookup (a chunk's last run may
            // stay partial)
            asm volatile(
                "{\n\t"
                ".reg .u32 plo, phi, x;\n\t"
                ".reg .pred dn;\n\t"
                "shf.l.wrap.b32 plo, 0, %4, %5;\n\t"
                "shf.l.wrap.b32 phi, %4, 0, %5;\n\t"
                "mad.lo.u32 %0, plo, %6, %0;\n\t"
                "st.shared.u32 [%2], %0;\n\t"
                "and.b32 x, %1, 0x2000;\n\t"
                "setp.ne.u32 dn, x, 0;\n\t"
                "selp.b32 %0, phi, %0, dn;\n\t"
                "@dn mad.lo.u32 %1, %6, %7, %1;\n\t"
                "@dn mad.lo.u32 %2, %6, %3, %2;\n\t"
                "}"
                : "+r"(p0), "+r"(C), "+r"(osta)
                : "r"(kRunBytes), "r"(codes), "r"(q), "r"(k.one), "r"(0xE000u)
                : "memory");
        } else if (RING == 0) {
            // pending bits < 64 before the append: below bit 32 of the string the codes
            // go to p0 and what passes bit 32 to p1 (then zero); above, to p1 and past bit 64
            // (phi) to the next run; the run's two words are stored once, when it is whole
            asm volatile(
                "{\n\t"
                ".reg .u32 plo, phi, x;\n\t"
                ".reg .pred hs, dn;\n\t"
                "shf.l.wrap.b32 plo, 0, %5, %6;\n\t"
                "shf.l.wrap.b32 phi, %5, 0, %6;\n\t"
                "and.b32 x, %6, 32;\n\t"
                "setp.ne.u32 hs, x, 0;\n\t"
                "selp.b32 %1, %1, phi, hs;\n\t"
                "@!hs mad.lo.u32 %0, plo, %7, %0;\n\t"
                "@hs mad.lo.u32 %1, plo, %7, %1;\n\t"
                "and.b32 x, %2, 0x4000;\n\t"
                "setp.ne.u32 dn, x, 0;\n\t"
                "@dn st.shared.v2.u32 [%3], {%0, %1};\n\t"
                "selp.b32 %0, phi, %0, dn;\n\t"
                "selp.b32 %1, 0, %1, dn;\n\t"
                "@dn mad.lo.u32 %2, %7, %8, %2;\n\t"  // runs + 1, pending - 64
                "@dn mad.lo.u32 %3, %7, %4, %3;\n\t"
                "}"
                : "+r"(p0), "+r"(p1), "+r"(C), "+r"(osta)
                : "r"(kRunBytes), "r"(codes), "r"(q), "r"(k.one), "r"(0xC000u)
                : "memory");
        } else {
            // pending bits < 64 before the append: below bit 32 of the string the codes
            // go to p0 and what passes bit 32 to p1 (then zero); above, to p1 and past bit 64
            // (phi) to the next run; a ring's slot holds the run so far after every lookup
            asm volatile(
                "{\n\t"
                ".reg .u32 plo, phi, x;\n\t"
                ".reg .pred hs, dn;\n\t"
                "shf.l.wrap.b32 plo, 0, %5, %6;\n\t"
                "shf.l.wrap.b32 phi, %5, 0, %6;\n\t"
                "and.b32 x, %6, 32;\n\t"
                "setp.ne.u32 hs, x, 0;\n\t"
                "selp.b32 %1, %1, phi, hs;\n\t"
                "@!hs mad.lo.u32 %0, plo, %7, %0;\n\t"
                "@hs mad.lo.u32 %1, plo, %7, %1;\n\t"
                "st.shared.v2.u32 [%3], {%0, %1};\n\t"
                "and.b32 x, %2, 0x4000;\n\t"
                "setp.ne.u32 dn, x, 0;\n\t"
                "selp.b32 %0, phi, %0, dn;\n\t"
                "selp.b32 %1, 0, %1, dn;\n\t"
                "@dn mad.lo.u32 %2, %7, %8, %2;\n\t"  // runs + 1, pending - 64
                "@dn mad.lo.u32 %3, %7, %4, %3;\n\t"
                "}"
                : "+r"(p0), "+r"(p1), "+r"(C), "+r"(osta)
                : "r"(kRunBytes), "r"(codes), "r"(q), "r"(k.one), "r"(0xC000u)
                : "memory");
        }
        if (RING > 0) {
            // the slot after the ring's last is its first
            asm volatile(
                "{\n\t"
                ".reg .pred w;\n\t"
                "setp.ge.u32 w, %0, %1;\n\t"
                "@w sub.u32 %0, %0, %2;\n\t"
                "}"
                : "+r"(osta)
                : "r"(rend), "n"(RING * RB));
        }
    }
};

// Advance every lane the thread serves to at least run te, STEPS lookups per
// check, until every lane of the warp has reached te; a lane that is ahead
// keeps decoding up to run cap (the chunk's end).
template <int STEPS, int BITS, bool SLOW, int LANES, uint32_t RB, int RING, bool CO, int LPT>
__device__ __forceinline__ void wide_decode_to(WideDecoder<BITS, SLOW, LANES, RB, RING, CO> (&ld)[LPT],
                                               const Pipes &pk, const uint32_t *slim,
                                               const int32_t *soffs, const uint8_t *ssyms, int te, int cap,
                                               int max_len, bool refill_each, int32_t *status) {
    const uint32_t te_c = static_cast<uint32_t>(te) << kRunsShift, cap_c = static_cast<uint32_t>(cap) << kRunsShift;
    for (;;) {
        bool behind = false;
#pragma unroll
        for (int k = 0; k < LPT; k++) behind = behind || ld[k].C < te_c;
        if (!__any_sync(0xffffffffu, behind)) break;
        // refill points: after every second lookup, or after every lookup when refill_each
        const bool r0 = SLOW && refill_each;
        if (CO) {
            // the refills' ballot needs the whole warp: a lane at its chunk's end runs
            // no-op lookups (and, having no words left, takes none)
            static_assert(!CO || LPT == 1, "consumption order: one lane per thread");
            const bool live = ld[0].C < cap_c;
#pragma unroll
            for (int h = 0; h < STEPS / 2; h++) {
                ld[0].step(pk, r0, slim, soffs, ssyms, max_len, status, live);
                ld[0].step(pk, true, slim, soffs, ssyms, max_len, status, live);
            }
        } else if (LPT == 1) {
            if (ld[0].C < cap_c) {
#pragma unroll
                for (int h = 0; h < STEPS / 2; h++) {
                    ld[0].step(pk, r0, slim, soffs, ssyms, max_len, status);
                    ld[0].step(pk, true, slim, soffs, ssyms, max_len, status);
                }
            }
        } else {
            // several streams per thread: their lookups interleave (independent chains)
            bool live[LPT];
#pragma unroll
            for (int k = 0; k < LPT; k++) live[k] = ld[k].C < cap_c;
#pragma unroll
            for (int h = 0; h < STEPS / 2; h++) {
#pragma unroll
                for (int k = 0; k < LPT; k++) ld[k].step(pk, r0, slim, soffs, ssyms, max_len, status, live[k]);
#pragma unroll
                for (int k = 0; k < LPT; k++) ld[k].step(pk, true, slim, soffs, ssyms, max_len, status, live[k]);
            }
        }
    }
}

