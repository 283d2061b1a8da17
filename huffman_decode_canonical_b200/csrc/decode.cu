// decode.cu -- sm_100a kernels and the device half of the libentro C ABI.
//
// What runs here (EntroLLM, arXiv 2505.02380v4, abstract and "parallel
// decoding" in the technical summary; LazyWeights, arXiv 2611.17108v1,
// abstract: interleaved lanes, decode on demand so memory moves only coded
// bytes):
//   * lanes kernel: one warp per chunk of the interleaved-lane format (32 or
//     64 lanes; a thread serves one or two lanes).  The chunk's words are
//     staged into shared memory with cp.async.bulk (one elected lane,
//     mbarrier completion, double buffered per warp, a copy per CTA).  Each
//     lane decodes with the two-word-table decoder of wide_decoder.cuh (up to
//     eight 4-bit or four 8-bit codes per 12-bit peek, canonical length tables
//     for codes longer than 12 bits) into a 16-run ring.  Lane l emits runs of
//     8 adjacent weights, so a warp writes 128/256/512 contiguous bytes per
//     run (uint4 codes / uint8 codes / bf16) with one vector store per lane.
//   * rows kernel (rows.cuh): the row-tile format, lane = row of a tile; codes,
//     bf16 and the fused GEMV on the tensor cores at every batch size.
//   * the same kernel dequantizes, w = bf16_rne(float(q - zero) * scale), with
//     the value of every code computed once per CTA in fp32 and looked up in
//     a shared-memory table (for 4-bit codes, by byte: two values per entry),
//     or feeds the bf16 weights straight into an fp32 GEMV with a
//     warp-shuffle reduction per row (weights never touch memory).
//   * gemv_mma kernel: the lanes format's fused GEMV for batches of 3 to 16
//     activation rows.  The warps of a CTA decode consecutive rows in lockstep
//     (one-word multi-symbol table, up to six 4-bit or three 8-bit codes per
//     peek) and multiply the decoded weights with warp-level tensor-core MMAs
//     (mma.sync m16n8k16, bf16 in, fp32 out), reading the A operand from the
//     warps' code rings.
//   * segment kernel: the one-bitstream-per-chunk format, one CTA per chunk
//     of up to 16384 codes.  Its threads decode segments cut at 32-bit
//     boundaries, re-decode from where the left neighbour stopped until they
//     meet a code start they marked (Huffman codes resynchronise within a
//     few codes), place their codes with a block-wide scan and write them
//     through shared memory.
//   * single kernel: the same format with larger chunks, one thread per chunk.
// The decode itself is bit manipulation and streaming, not a dense
// contraction; only the batched GEMV is MMA-shaped.  Errors are reported
// through a status word, never by trapping; every wait on a copy is bounded.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "blob_format.h"
#include "entro.h"
#include "entro_internal.h"

namespace entro {

constexpr int kLutSize = 1 << kMaxLutBits;   // 4096 entries, 16 KB of shared memory
constexpr int kWideLutBytes = kLutSize * 8;  // the two-word table: 4096 entries of {codes, meta}
constexpr long long kWaitCycles = 1LL << 31;  // ~1 s at B200 clocks
constexpr int kMaxWarps = 16;
constexpr int kMaxBatch = 16;
constexpr int kSlackRows = 2;                 // staging rows past a chunk's longest lane (read-ahead)
// A lane's window may run past its last word by the lookups made after its last
// run completes (up to 5 of at most 24 bits, plus the word loaded one ahead):
// reads stay inside the staging buffer (clamped); a lane that moved more than
// this many rows past its words has decoded a corrupt stream.
constexpr int kOverrunRows = 7;

enum OutKind { OUT_CODES = 0, OUT_BF16 = 1, OUT_GEMV = 2 };

struct DevTensor {
    const uint32_t *lut;         // [4096] one code per entry: length | symbol << 8
    const uint32_t *mlut;        // [4096] several codes per entry: bits | count << 4 | symbols << 8
    const uint32_t *slow_limit;  // [32]  (first[l] + count[l]) << (max_len - l)
    const int32_t *slow_offs;    // [32]  rank of the first code of length l minus first[l]
    const uint8_t *slow_syms;    // [256] symbols sorted by (length, symbol)
    const uint2 *wlut;           // [4096] {codes, meta}: up to 8 (4-bit) or 4 (8-bit) codes per entry
    const uint64_t *index;       // (n_chunks + 1) x {start, first_symbol}
    const uint32_t *payload;
    long long n, rows, cols, chunk_symbols, n_chunks, payload_words;
    float scale;
    int zero, bits, max_len, format, max_chunk_words, n_codes, lanes;
};

struct GroupEntry {
    DevTensor d;
    void *out;               // codes or bf16 output
    const __nv_bfloat16 *x;  // GEMV input [batch, cols]
    float *y;                // GEMV output [batch, rows]
    long long chunk_begin;   // prefix over entries, in chunks
    long long sym_begin;     // prefix over entries, in symbols
};

static_assert(sizeof(GroupEntry) == 184, "the fixed group table is documented as 184-byte entries");

struct LaunchArgs {
    const GroupEntry *table;  // device array, or nullptr: use `one`
    GroupEntry one;
    int count;
    int batch;
    int x_in_smem;
    int stage_rows;       // rows of 32 words per staging buffer (longest chunk + slack)
    int out_words;        // per-warp code staging, 32-bit words
    long long x_elems;    // bf16 activations held in shared memory
    long long total_syms;
    int32_t *status;
    uint32_t tx_extra;    // bytes added to the table barrier that never arrive (bounded-wait test; 0)
    uint32_t k_one;       // 1, a value the compiler cannot see (moves integer work to the FMA pipe)
};

struct TensorHandle {
    DevTensor d;
    int device;
    bool slow;
    uint64_t device_bytes;
};

// ------------------------------------------------------------------ device helpers

// Programmatic dependent launch: a launch made with the overlap attribute may
// start while the kernel before it on the stream is finishing.  A kernel lets
// the next launch begin at once (it cannot take this kernel's SM resources
// before they are freed), reads only the tensors' device images before
// grid_wait_prior(), and touches activations, outputs and the status word only
// after it.  Both are no-ops for a launch without the attribute.
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_wait_prior() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void set_status(int32_t *st, int code) {
    if (st) atomicCAS(st, 0, code);
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

// Bulk global -> shared copy completing on an mbarrier (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: gives up after ~1 s instead of hanging the GPU.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > kWaitCycles) return false;
    return true;
}

// acc += lo(w2) * lo(x2), then acc += hi(w2) * hi(x2): bf16 operands, fp32
// accumulation with one rounding per step (the same value as an fp32 FMA of
// the widened operands).
__device__ __forceinline__ float fma2_bf16(uint32_t w2, uint32_t x2, float acc) {
    asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
        "mov.b32 {wl, wh}, %1;\n\t"
        "mov.b32 {xl, xh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, wl, xl, %0;\n\t"
        "fma.rn.f32.bf16 %0, wh, xh, %0;\n\t}"
        : "+f"(acc)
        : "r"(w2), "r"(x2));
    return acc;
}

// Canonical decode of a code longer than the table's 12 bits: the code length
// is the first l with (top max_len bits) < limit[l].  Returns length | symbol
// << 8, or a 1-bit entry after flagging corruption.
__device__ __forceinline__ uint32_t slow_entry(uint64_t win, int max_len, const uint32_t *limit,
                                            const int32_t *offs, const uint8_t *syms, int32_t *status) {
    const uint32_t v = static_cast<uint32_t>(win >> (64 - max_len));
    int l = kMaxLutBits + 1;
    while (l <= max_len && v >= limit[l]) l++;
    if (l > max_len) {
        set_status(status, ENTRO_E_CORRUPT);
        return 1u;
    }
    const uint32_t sym = syms[(offs[l] + static_cast<int>(v >> (max_len - l))) & 255];
    return static_cast<uint32_t>(l) | (sym << 8);
}

struct Smem {
    uint32_t *lut;    // decode table (multi-symbol for the lanes kernel)
    uint32_t *vtab;   // bf16 value of each code, low half
    uint32_t *vpair;  // 4-bit: bf16 values of the two codes of a byte
    uint32_t *slim;
    int32_t *soffs;
    uint8_t *ssyms;
    __nv_bfloat16 *xs;
    uint64_t *tbar;   // CTA barrier for the table copies
    uint64_t *bars;
    uint32_t *stage;
    uint32_t *ostage;
    float *red;       // tensor-core GEMV: per-warp partial sums for the cross-warp row reduction
};

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct SmemOffsets {
    size_t x, bars, stage, ostage, red, total;
};

// shared-memory carve-up; identical on host (sizing) and device
// stage_words: 32-bit words of one staging buffer (rows x lanes); red_bytes:
// the cross-warp partial sums of the tensor-core GEMV
// lut_bytes: the decode table (kLutSize * 4, or * 8 for the two-word table)
__host__ __device__ inline SmemOffsets smem_layout(int warps, long long x_elems, int stage_words, int out_words,
                                                   size_t red_bytes = 0, size_t lut_bytes = kLutSize * 4) {
    SmemOffsets o;
    size_t p = lut_bytes + 256 * 4 + 256 * 4 + 32 * 4 + 32 * 4 + 256;
    p = align_up(p, 16);
    o.x = p;
    p += (size_t)x_elems * 2;
    p = align_up(p, 16);
    o.bars = p;
    p += (size_t)(warps + 1) * 2 * 8;
    p = align_up(p, 128);
    o.stage = p;
    p += (size_t)warps * 2 * (size_t)stage_words * 4;
    p = align_up(p, 16);
    o.ostage = p;
    p += (size_t)warps * (size_t)out_words * 4;
    p = align_up(p, 16);
    o.red = p;
    p += red_bytes;
    o.total = p;
    return o;
}

__device__ __forceinline__ Smem carve(uint8_t *base, int warps, long long x_elems, int stage_words, int out_words,
                                      size_t red_bytes = 0, size_t lut_bytes = kLutSize * 4) {
    const SmemOffsets o = smem_layout(warps, x_elems, stage_words, out_words, red_bytes, lut_bytes);
    Smem s;
    s.lut = reinterpret_cast<uint32_t *>(base);
    s.vtab = s.lut + lut_bytes / 4;
    s.vpair = s.vtab + 256;
    s.slim = s.vpair + 256;
    s.soffs = reinterpret_cast<int32_t *>(s.slim + 32);
    s.ssyms = reinterpret_cast<uint8_t *>(s.soffs + 32);
    s.xs = reinterpret_cast<__nv_bfloat16 *>(base + o.x);
    s.tbar = reinterpret_cast<uint64_t *>(base + o.bars);
    s.bars = s.tbar + 2;
    s.stage = reinterpret_cast<uint32_t *>(base + o.stage);
    s.ostage = reinterpret_cast<uint32_t *>(base + o.ostage);
    s.red = reinterpret_cast<float *>(base + o.red);
    return s;
}

__device__ __forceinline__ uint32_t dequant_bf16_bits(int q, int zero, float scale) {
    const float f = __fmul_rn(__int2float_rn(q - zero), scale);
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

// The 4-bit value-pair table (the bf16 values of both codes of a byte) is stored
// at a swizzled index: bits 5..7 of the byte (the high code's upper three bits)
// are XORed into bits 2..4.  A warp's 32 lookups take bytes of 32 different
// runs; with the plain index a byte's bank is its low code and the high code's
// lowest bit, so the frequent high codes 6, 8, 10 (or 7, 9) of a centred
// 4-bit distribution share banks.  The swizzle is a bijection and keeps the
// table at 256 words; one shift and one LOP3 swizzle all four bytes of a slot.
__host__ __device__ constexpr uint32_t vpair_index(uint32_t b) { return b ^ ((b >> 3) & 0x1Cu); }
__device__ __forceinline__ uint32_t vpair_swizzle4(uint32_t c) { return c ^ ((c >> 3) & 0x1C1C1C1Cu); }

// Per-tensor tables into shared memory.  vtab[q] is the dequantized weight
// bf16_rne(float(q - zero) * scale) (EntroLLM: weights are kept as quantized
// codes and dequantized for inference), computed here in fp32 once per CTA;
// vpair[vpair_index(b)] holds the values of both 4-bit codes of byte b.  The decode table,
// the canonical tables and (GEMV) the activations arrive by bulk copies on the
// CTA barrier; thread 0 issues them at phase `tphase`.
// table: 0 = one code per entry (lut), 1 = several (mlut), 2 = the two-word table (wlut)
template <int OUT, bool SLOW>
__device__ void issue_tables(const GroupEntry &g, const Smem &s, int table, int batch, int x_in_smem,
                             uint32_t tx_extra) {
    if (threadIdx.x != 0) return;
    const DevTensor &d = g.d;
    const uint32_t tbytes = table == 2 ? kWideLutBytes : kLutSize * 4;
    uint32_t bytes = tbytes + tx_extra;
    if (SLOW) bytes += kSlowBytes;
    const uint32_t xbytes = (OUT == OUT_GEMV && x_in_smem) ? static_cast<uint32_t>(d.cols * batch * 2) : 0u;
    bytes += xbytes;
    mbar_arrive_expect_tx(s.tbar, bytes);
    const void *src = table == 2 ? static_cast<const void *>(d.wlut) : table == 1 ? d.mlut : d.lut;
    bulk_copy_g2s(s.lut, src, tbytes, s.tbar);
    if (SLOW) bulk_copy_g2s(s.slim, d.slow_limit, kSlowBytes, s.tbar);
}

// The activations' copy, counted on the same barrier by issue_tables; issued
// after grid_wait_prior(), since the kernel before may be writing them.
template <int OUT>
__device__ void issue_x(const GroupEntry &g, const Smem &s, int batch, int x_in_smem) {
    if (threadIdx.x != 0 || OUT != OUT_GEMV || !x_in_smem) return;
    bulk_copy_g2s(s.xs, g.x, static_cast<uint32_t>(g.d.cols * batch * 2), s.tbar);
}

template <int OUT, bool SLOW>
__device__ bool finish_tables(const GroupEntry &g, const Smem &s, uint32_t tphase) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const DevTensor &d = g.d;
    if (OUT != OUT_CODES) {
        for (int q = tid; q < 256; q += nthr) {
            const uint32_t v = q < (1 << d.bits) ? dequant_bf16_bits(q, d.zero, d.scale) : 0u;
            s.vtab[q] = v;
            if (d.bits == 4)
                s.vpair[vpair_index(q)] = dequant_bf16_bits(q & 15, d.zero, d.scale) |
                             (dequant_bf16_bits(q >> 4, d.zero, d.scale) << 16);
        }
    }
    const bool ok = mbar_wait(s.tbar, tphase & 1);
    __syncthreads();
    return __syncthreads_and(ok);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ------------------------------------------------------------------ phase 1: one lane's stream
//
// The lane keeps a 64-bit MSB-first window of its bitstream.  One 12-bit peek
// into the multi-symbol table yields up to 6 (4-bit) or 3 (8-bit) symbols and
// the bits they take; codes longer than 12 bits go through the canonical
// slow path.  Symbols collect in a pending register; every 8 form one run,
// written to the warp's code stage at word 32*t + lane (4-bit) or double-word
// 32*t + lane (8-bit), i.e. in output order, without bank conflicts.

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void sts64(uint32_t addr, uint32_t lo, uint32_t hi) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(lo), "r"(hi) : "memory");
}

// Runs are staged in a ring of kRing slots per lane; the slot of run t is
// written while run t is being assembled.  A check of a lane's progress is
// followed by kLookupsPerCheck lookups of at most kMaxCodesPerLookup codes
// each, which, with at most kRun - 1 codes pending, complete at most
// kRunsPerCheck runs.  The lanes kernel emits every kEmitBlock runs and lets a
// lane decode up to kLookahead runs into the next block, so the slots in use
// while a block waits to be emitted are kEmitBlock + kLookahead +
// kRunsPerCheck <= kRing.
constexpr int kEmitBlock = 8;
constexpr int kRing = 16;
constexpr int kMaxCodesPerLookup = 6;  // multi-symbol table: up to 6 4-bit or 3 8-bit codes per entry
__host__ __device__ constexpr int runs_per_check(int lookups) {
    return (kRun - 1 + lookups * kMaxCodesPerLookup) / kRun;
}
constexpr int kLookupsPerCheck = 6;    // lanes kernel: table lookups between two checks of a lane's run count
// the lanes kernel's two-word decoder: 6 lookups per check for 4-bit codes (up to 8 per
// lookup, so the ring holds the overshoot), 8 for 8-bit codes (up to 4 per lookup)
template <int BITS>
__host__ __device__ constexpr int wide_lookups_per_check() { return BITS == 8 ? 8 : kLookupsPerCheck; }
constexpr int kRunsPerCheck = runs_per_check(kLookupsPerCheck);
constexpr int kLookahead = 3;          // lanes kernel: runs a lane may decode ahead into the next block
static_assert(kRing >= kEmitBlock + kLookahead + kRunsPerCheck, "ring too small for the decode overshoot");
constexpr int kTileLookupsPerCheck = 4;  // tensor-core GEMV kernel (longer lockstep blocks fit the ring)

// Shifts that give 0 for a shift of 32 (PTX clamps the amount to the width).
__device__ __forceinline__ uint32_t shl_clamp(uint32_t v, uint32_t n) {
    uint32_t r;
    asm("shl.b32 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(n));
    return r;
}
__device__ __forceinline__ uint32_t shr_clamp(uint32_t v, uint32_t n) {
    uint32_t r;
    asm("shr.b32 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(n));
    return r;
}

#include "wide_decoder.cuh"

template <int BITS, bool SLOW, int LANES>
struct LaneDecoder {
    static constexpr int kRunBits = 8 * BITS;
    static constexpr uint32_t kRowBytes = 4 * LANES;           // one staged word of every lane
    static constexpr uint32_t kRunStride = LANES * BITS;       // bytes between a lane's ring slots
    uint32_t lut;         // shared address of the decode table
    uint32_t bufa;        // shared address of this lane's next word; word j at word 0 + kRowBytes j
    uint32_t bufcap;      // shared address of the last readable word of this lane
    uint32_t ostb;        // shared address of this lane's slot 0 of the run ring
    uint32_t osta;        // shared address of this lane's current run slot
    int nb;               // valid bits in the window
    uint32_t wnext;       // the next word, loaded one refill ahead (off the window's dependency chain)
    uint32_t hi, lo;      // 64-bit window, MSB first: the next bits of the stream start at bit 31 of hi
    uint32_t p0, p1, p2;  // pending codes as one bit string, first code at bit 0 of p0
    int pb;               // pending bits (BITS per code); below one run whenever codes are appended
    int t;                // runs completed

    __device__ __forceinline__ void init(const Smem &s, const uint32_t *b, uint32_t *o, int cap) {
        lut = smem_addr(s.lut);
        bufa = smem_addr(b);
        bufcap = bufa + kRowBytes * static_cast<uint32_t>(cap);
        ostb = osta = smem_addr(o);
        hi = lds32(bufa);
        lo = lds32(bufa + kRowBytes);
        nb = 64;
        bufa += 2 * kRowBytes;
        wnext = lds32(min(bufa, bufcap));
        p0 = p1 = p2 = 0;
        pb = 0;
        t = 0;
    }

    // Top the window up to more than 32 bits: the next word lands right below
    // the nb valid bits.  Branch-free apart from the predicated load.
    __device__ __forceinline__ void refill() {
        const bool need = nb <= 32;
        const uint32_t n = static_cast<uint32_t>(nb);
        hi |= need ? shr_clamp(wnext, n) : 0u;
        lo |= need ? shl_clamp(wnext, 32u - n) : 0u;
        nb += need ? 32 : 0;
        bufa += need ? kRowBytes : 0u;
        if (need) wnext = lds32(min(bufa, bufcap));
    }

    // One table lookup that only appends its codes to the pending bit string
    // (no slot store): the tail of a partial last run, closed by close_run().
    __device__ __forceinline__ void lookup(const Smem &s, int max_len, int32_t *status) {
        const uint32_t e = lds32(lut + ((hi >> (32 - kMaxLutBits)) << 2));
        uint32_t syms = e >> 8, bits = e & 15u;
        // count * BITS straight from the entry's count field (bits 4..7)
        int add = static_cast<int>(BITS == 4 ? (e >> 2) & 0x3Cu : (e >> 1) & 0x78u);
        if (SLOW && add == 0) {
            const uint64_t win = (static_cast<uint64_t>(hi) << 32) | lo;
            const uint32_t se = slow_entry(win, max_len, s.slim, s.soffs, s.ssyms, status);
            bits = se & 31u;
            syms = (se >> 8) & 0xFFu;
            add = BITS;
        }
        hi = __funnelshift_l(lo, hi, bits);  // bits <= 24: the top 32 bits of (hi:lo) << bits
        lo <<= bits;
        nb -= static_cast<int>(bits);
        const int q = pb & 31;
        const uint32_t plo = syms << q, phi = __funnelshift_l(syms, 0u, q);  // (0:syms) << q, 24-bit codes
        if (BITS == 4 || pb < 32) {
            p0 |= plo;
            p1 |= phi;
        } else {
            p1 |= plo;
            p2 |= phi;
        }
        pb += add;
    }

    // One table lookup and its run bookkeeping.  The window shift, the append
    // of the entry's codes to the pending string, the slot store and the run
    // completion are one block of hand-written PTX; a miss in the table (a
    // code longer than 12 bits) goes through the canonical slow path and
    // re-enters as a one-code entry.
    __device__ __forceinline__ void step(const Smem &s, int max_len, int32_t *status) {
        uint32_t e = lds32(lut + ((hi >> (32 - kMaxLutBits)) << 2));
        uint32_t bits = e & 15u;
        if (SLOW && (e & 0xF0u) == 0) {
            const uint64_t win = (static_cast<uint64_t>(hi) << 32) | lo;
            const uint32_t se = slow_entry(win, max_len, s.slim, s.soffs, s.ssyms, status);
            bits = se & 31u;
            e = (1u << 4) | (se & 0xFF00u);
        }
        advance(e, bits);
    }

    // Consume `bits` of the window and append the entry's codes (count in bits
    // 4..7 of e, codes from bit 8); store the current run's slot; move to the
    // next slot when the run is whole.
    __device__ __forceinline__ void advance(uint32_t e, uint32_t bits) {
        if (BITS == 4) {
            // pb < 32 before the append (a run completes at 32 bits)
            asm volatile(
                "{\n\t"
                ".reg .u32 add, syms, plo, phi, tw;\n\t"
                ".reg .pred done;\n\t"
                "shf.l.wrap.b32 %0, %1, %0, %9;\n\t"
                "shl.b32 %1, %1, %9;\n\t"
                "sub.s32 %2, %2, %9;\n\t"
                "and.b32 add, %8, 240;\n\t"
                "shr.u32 add, add, 2;\n\t"
                "shr.u32 syms, %8, 8;\n\t"
                "shl.b32 plo, syms, %5;\n\t"
                "shf.l.wrap.b32 phi, syms, 0, %5;\n\t"
                "or.b32 %3, %3, plo;\n\t"
                "or.b32 %4, %4, phi;\n\t"
                "add.s32 %5, %5, add;\n\t"
                "st.shared.u32 [%7], %3;\n\t"
                "setp.ge.s32 done, %5, 32;\n\t"
                "selp.b32 %3, %4, %3, done;\n\t"
                "selp.b32 %4, 0, %4, done;\n\t"
                "@done sub.s32 %5, %5, 32;\n\t"
                "@done add.s32 %6, %6, 1;\n\t"
                "and.b32 tw, %6, 15;\n\t"
                "mad.lo.u32 %7, tw, %11, %10;\n\t"
                "}"
                : "+r"(hi), "+r"(lo), "+r"(nb), "+r"(p0), "+r"(p1), "+r"(pb), "+r"(t), "+r"(osta)
                : "r"(e), "r"(bits), "r"(ostb), "n"(kRunStride)
                : "memory");
        } else {
            // pb < 64 before the append; codes go to p0:p1 below bit 32 of the
            // string's current word, to p1:p2 above
            asm volatile(
                "{\n\t"
                ".reg .u32 add, syms, plo, phi, q, tw;\n\t"
                ".reg .pred lt, done;\n\t"
                "shf.l.wrap.b32 %0, %1, %0, %10;\n\t"
                "shl.b32 %1, %1, %10;\n\t"
                "sub.s32 %2, %2, %10;\n\t"
                "shr.u32 add, %9, 1;\n\t"
                "and.b32 add, add, 120;\n\t"
                "shr.u32 syms, %9, 8;\n\t"
                "and.b32 q, %6, 31;\n\t"
                "shl.b32 plo, syms, q;\n\t"
                "shf.l.wrap.b32 phi, syms, 0, q;\n\t"
                "setp.lt.s32 lt, %6, 32;\n\t"
                "@lt or.b32 %3, %3, plo;\n\t"
                "@lt or.b32 %4, %4, phi;\n\t"
                "@!lt or.b32 %4, %4, plo;\n\t"
                "@!lt or.b32 %5, %5, phi;\n\t"
                "add.s32 %6, %6, add;\n\t"
                "st.shared.v2.u32 [%8], {%3, %4};\n\t"
                "setp.ge.s32 done, %6, 64;\n\t"
                "selp.b32 %3, %5, %3, done;\n\t"
                "selp.b32 %4, 0, %4, done;\n\t"
                "selp.b32 %5, 0, %5, done;\n\t"
                "@done sub.s32 %6, %6, 64;\n\t"
                "@done add.s32 %7, %7, 1;\n\t"
                "and.b32 tw, %7, 15;\n\t"
                "mad.lo.u32 %8, tw, %12, %11;\n\t"
                "}"
                : "+r"(hi), "+r"(lo), "+r"(nb), "+r"(p0), "+r"(p1), "+r"(p2), "+r"(pb), "+r"(t), "+r"(osta)
                : "r"(e), "r"(bits), "r"(ostb), "n"(kRunStride)
                : "memory");
        }
    }

    // store the current (possibly partial) run and count it done
    __device__ __forceinline__ void close_run() {
        if (BITS == 4) sts32(osta, p0);
        else sts64(osta, p0, p1);
        t++;
        osta = ostb + static_cast<uint32_t>(t & (kRing - 1)) * kRunStride;
    }
};

// ------------------------------------------------------------------ phase 2: stage -> output

// 8 codes of run-word w -> 8 bf16 values (4 words, value of code 8w+i in half i)
template <int BITS>
__device__ __forceinline__ uint4 values8(const Smem &s, const uint32_t *ost, int w) {
    uint4 v;
    if (BITS == 4) {
        const uint32_t c = vpair_swizzle4(ost[w]);
        v.x = s.vpair[c & 0xFFu];
        v.y = s.vpair[(c >> 8) & 0xFFu];
        v.z = s.vpair[(c >> 16) & 0xFFu];
        v.w = s.vpair[c >> 24];
    } else {
        const uint2 c = reinterpret_cast<const uint2 *>(ost)[w];
        v.x = __byte_perm(s.vtab[c.x & 0xFFu], s.vtab[(c.x >> 8) & 0xFFu], 0x5410);
        v.y = __byte_perm(s.vtab[(c.x >> 16) & 0xFFu], s.vtab[c.x >> 24], 0x5410);
        v.z = __byte_perm(s.vtab[c.y & 0xFFu], s.vtab[(c.y >> 8) & 0xFFu], 0x5410);
        v.w = __byte_perm(s.vtab[(c.y >> 16) & 0xFFu], s.vtab[c.y >> 24], 0x5410);
    }
    return v;
}

// Emit runs [tb, te) of a whole chunk (every lane owns 8 codes per run);
// thread `lane` serves the format lanes lane, lane + 32, ...
template <int BITS, int OUT, int BPAD, int LANES>
__device__ __forceinline__ void emit_runs(const GroupEntry &g, const Smem &s, const uint32_t *ost, long long first,
                                          int tb, int te, int batch, int x_in_smem, float (&acc)[BPAD],
                                          int &st, long long &row) {
    constexpr int LPT = LANES / kLanes;
    const DevTensor &d = g.d;
    const int lane = threadIdx.x & 31;
    if (OUT == OUT_CODES) {
        // staged codes are packed and in output order (the block's slots do not wrap): 16-byte copies
        constexpr int kU4PerRun = LANES * BITS / 16;  // uint4 per run of the chunk
        const uint4 *src = reinterpret_cast<const uint4 *>(ost) + (tb & (kRing - 1)) * kU4PerRun;
        uint4 *dst = reinterpret_cast<uint4 *>(g.out) + first * BITS / 128 + tb * kU4PerRun;
        for (int i = lane; i < (te - tb) * kU4PerRun; i += kLanes) dst[i] = src[i];
    } else if (OUT == OUT_BF16) {
        // four runs per pass: their table lookups are all in flight before the stores
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(g.out) + first);
        int t = tb;
        for (; t + 4 <= te; t += 4) {
            uint4 v[4][LPT];
#pragma unroll
            for (int j = 0; j < 4; j++)
#pragma unroll
                for (int k = 0; k < LPT; k++)
                    v[j][k] = values8<BITS>(s, ost, LANES * ((t + j) & (kRing - 1)) + lane + kLanes * k);
#pragma unroll
            for (int j = 0; j < 4; j++)
#pragma unroll
                for (int k = 0; k < LPT; k++) dst[LANES * (t + j) + lane + kLanes * k] = v[j][k];
        }
        for (; t < te; t++)
#pragma unroll
            for (int k = 0; k < LPT; k++) {
                const int l = lane + kLanes * k;
                dst[LANES * t + l] = values8<BITS>(s, ost, LANES * (t & (kRing - 1)) + l);
            }
    } else {
        // fused GEMV (batch 1 and 2): run t covers columns 8*LANES*(t % spr) + 8*l .. +7
        // of row t / spr.  Four runs per pass: each run's 8 weights are
        // multiplied with mixed-precision FMAs of the bf16 weights and
        // activations (fma.rn.f32.bf16) into a partial sum of its own, so the
        // passes' loads and FMA chains overlap; the partials are then added to
        // the lane's row sum in run order, and the warp reduces at the row end.
        // `st` (run step within the row) and `row` carry over from block to block.
        const int K = static_cast<int>(d.cols);
        const int spr = K / (kRun * LANES);
        const int xrow = K >> 3;  // uint4 per row of x
        const uint4 *xg = reinterpret_cast<const uint4 *>(g.x);
        const uint4 *xsm = reinterpret_cast<const uint4 *>(s.xs);
        for (int t = tb; t < te; t += 4) {
            const int n = min(4, te - t);
            int stj[4];
            {
                int sj = st;
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    stj[j] = sj;
                    sj = sj + 1 == spr ? 0 : sj + 1;
                }
                st = stj[0];
#pragma unroll
                for (int j = 0; j < 4; j++)
                    if (j < n) st = st + 1 == spr ? 0 : st + 1;
            }
            float part[4][BPAD];
#pragma unroll
            for (int j = 0; j < 4; j++) {
#pragma unroll
                for (int b = 0; b < BPAD; b++) part[j][b] = 0.f;
                if (j < n) {
#pragma unroll
                    for (int k = 0; k < LPT; k++) {
                        const int l = lane + kLanes * k;
                        const uint4 wv = values8<BITS>(s, ost, LANES * ((t + j) & (kRing - 1)) + l);
                        const int xo = stj[j] * LANES + l;
#pragma unroll
                        for (int b = 0; b < BPAD; b++) {
                            if (b < batch) {
                                const int xi = b * xrow + xo;
                                const uint4 xv = x_in_smem ? xsm[xi] : __ldg(xg + xi);
                                float p = part[j][b];
                                p = fma2_bf16(wv.x, xv.x, p);
                                p = fma2_bf16(wv.y, xv.y, p);
                                p = fma2_bf16(wv.z, xv.z, p);
                                p = fma2_bf16(wv.w, xv.w, p);
                                part[j][b] = p;
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < 4; j++) {
                if (j < n) {
#pragma unroll
                    for (int b = 0; b < BPAD; b++) acc[b] += part[j][b];
                    if (stj[j] == spr - 1) {
#pragma unroll
                        for (int b = 0; b < BPAD; b++) {
                            if (b < batch) {
                                const float v = warp_sum(acc[b]);
                                if (lane == 0) g.y[static_cast<long long>(b) * d.rows + row] = v;
                            }
                            acc[b] = 0.f;
                        }
                        row++;
                    }
                }
            }
        }
    }
}

// Emit runs [tb, te) of a ragged (last) chunk of nc codes: only positions < nc.
template <int BITS, int OUT, int LANES>
__device__ __forceinline__ void emit_ragged(const GroupEntry &g, const Smem &s, const uint32_t *ost, long long first,
                                            int nc, int tb, int te) {
    constexpr int LPT = LANES / kLanes;
    const int lane = threadIdx.x & 31;
    for (int t = tb; t < te; t++) {
        for (int k = 0; k < LPT; k++) {
            const int l = lane + kLanes * k;
            const int w = LANES * t + l;            // output word: positions 8w .. 8w+7
            const int cnt = min(8, nc - 8 * w);
            if (cnt <= 0) continue;
            const int slot = LANES * (t & (kRing - 1)) + l;
            if (OUT == OUT_CODES) {
                uint8_t *o = reinterpret_cast<uint8_t *>(g.out) + first * BITS / 8;
                if (BITS == 4) {
                    const uint32_t c = ost[slot];
                    for (int q = 0; 2 * q < cnt; q++) {
                        uint32_t b = (c >> (8 * q)) & 0xFFu;
                        if (2 * q + 1 >= cnt) b &= 0xFu;
                        o[4 * w + q] = static_cast<uint8_t>(b);
                    }
                } else {
                    const uint8_t *c = reinterpret_cast<const uint8_t *>(ost) + 8 * slot;
                    for (int q = 0; q < cnt; q++) o[8 * w + q] = c[q];
                }
            } else if (OUT == OUT_BF16) {
                const uint4 v = values8<BITS>(s, ost, slot);
                uint16_t *o = reinterpret_cast<uint16_t *>(g.out) + first + 8 * w;
                if (cnt == 8) {
                    *reinterpret_cast<uint4 *>(o) = v;
                } else {
                    for (int q = 0; q < cnt; q++) {
                        const uint32_t pair = (q < 2) ? v.x : (q < 4) ? v.y : (q < 6) ? v.z : v.w;
                        o[q] = static_cast<uint16_t>(pair >> (16 * (q & 1)));
                    }
                }
            }
        }
    }
}

// Advance every format lane the thread serves to at least run te (whole
// runs), STEPS lookups per check, until every lane of the warp has reached
// te.  Meanwhile a lane that is ahead keeps decoding up to run cap (>= te):
// work of the next block instead of idling while the warp's slowest lane
// finishes.  A lane may complete up to runs_per_check(STEPS) runs past the
// check that stops it, and read past its last word by up to STEPS - 1
// lookups (clamped to the staging buffer).
template <int STEPS, int BITS, bool SLOW, int LANES, int LPT>
__device__ __forceinline__ void decode_to(LaneDecoder<BITS, SLOW, LANES> (&ld)[LPT], const Smem &s, int te,
                                          int cap, int max_len, bool refill_each, int32_t *status) {
    for (;;) {
        bool behind = false;
#pragma unroll
        for (int k = 0; k < LPT; k++) behind = behind || ld[k].t < te;
        if (!__any_sync(0xffffffffu, behind)) break;
#pragma unroll
        for (int k = 0; k < LPT; k++) {
            if (ld[k].t < cap) {
#pragma unroll
                for (int h = 0; h < STEPS / 2; h++) {
                    ld[k].refill();
                    ld[k].step(s, max_len, status);
                    if (SLOW && refill_each) ld[k].refill();
                    ld[k].step(s, max_len, status);
                }
            }
        }
    }
}

// The lanes kernel's decoder: the two-word table, run slots in the warp's
// ring (run t of lane l in slot t mod kRing, word (t mod kRing) * LANES + l
// for 4-bit codes, double-word for 8-bit).  Lanes that finish a block decode
// up to kWideLookahead runs of the next; a block, the lookahead and the runs a
// lane may complete past its last check fit the ring.
template <int BITS>
__host__ __device__ constexpr int wide_lookahead() {
    return kRing - kEmitBlock - wide_runs_per_check(BITS, wide_lookups_per_check<BITS>()) < 3
               ? kRing - kEmitBlock - wide_runs_per_check(BITS, wide_lookups_per_check<BITS>())
               : 3;
}
static_assert(wide_lookahead<4>() >= 1 && wide_lookahead<8>() >= 1, "ring too small for the wide decoder");
template <int BITS, bool SLOW, int LANES>
using RingDecoder = WideDecoder<BITS, SLOW, LANES, LANES * (BITS == 4 ? 4u : 8u), kRing>;

// Decode chunk c of entry g from its staged words.  Thread `lane` decodes the
// format lanes lane, lane + 32, ... as independent interleaved streams.  Whole
// chunks are emitted every kEmitBlock runs, so the stores of one block drain
// while the lanes decode the next.
template <int BITS, int OUT, bool SLOW, int BPAD, int LANES>
__device__ __forceinline__ void decode_chunk(const GroupEntry &g, const Smem &s, const Pipes &pk,
                                             const uint32_t *buf, uint32_t *ost, int stage_rows, long long c,
                                             int batch, int x_in_smem, int32_t *status) {
    constexpr int LPT = LANES / kLanes;
    constexpr int kStep = kRun * LANES;  // symbols per lane step
    const DevTensor &d = g.d;
    const int lane = threadIdx.x & 31;
    const long long st = static_cast<long long>(d.index[2 * c]);
    const long long nx = static_cast<long long>(d.index[2 * c + 2]);
    const int words = static_cast<int>((nx - st) / LANES);
    const long long first = c * d.chunk_symbols;
    const long long remain = d.n - first;
    const int nc = static_cast<int>(remain < d.chunk_symbols ? remain : d.chunk_symbols);
    const bool refill_each = SLOW && d.max_len > 16;
    RingDecoder<BITS, SLOW, LANES> ld[LPT];
    uint32_t read_limit[LPT];
#pragma unroll
    for (int k = 0; k < LPT; k++) {
        const int l = lane + kLanes * k;
        ld[k].init(pk, smem_addr(s.lut), smem_addr(buf + l), smem_addr(ost + (BITS == 4 ? l : 2 * l)),
                   stage_rows - 1, true);
        // a valid lane never moves more than kOverrunRows rows past its words
        read_limit[k] = smem_addr(buf + l) + 4u * LANES * static_cast<uint32_t>(words + kOverrunRows);
    }
    bool ok = true;
    if (nc % kStep == 0) {
        // whole runs in every lane: every chunk but a short last one, and any
        // last chunk of whole rows (the GEMV's chunks always are)
        const int runs = nc / kStep;
        float acc[BPAD];
#pragma unroll
        for (int b = 0; b < BPAD; b++) acc[b] = 0.f;
        // GEMV: run step within the row and the row of the chunk's first run (chunks are whole rows)
        int gst = 0;
        long long grow = OUT == OUT_GEMV ? c * static_cast<long long>(static_cast<int>(d.chunk_symbols) /
                                                                      static_cast<int>(d.cols))
                                         : 0;
        for (int tb = 0; tb < runs; tb += kEmitBlock) {
            const int te = min(tb + kEmitBlock, runs);
            // a lane may run up to wide_lookahead runs into the next block, never past the chunk
            wide_decode_to<wide_lookups_per_check<BITS>()>(ld, pk, s.slim, s.soffs, s.ssyms, te,
                                             te < runs ? te + wide_lookahead<BITS>() : te, d.max_len, refill_each,
                                             status);
            __syncwarp();
            emit_runs<BITS, OUT, BPAD, LANES>(g, s, ost, first, tb, te, batch, x_in_smem, acc, gst, grow);
            __syncwarp();  // the ring slots just read are rewritten by the next block
        }
#pragma unroll
        for (int k = 0; k < LPT; k++) ok = ok && ld[k].bufa <= read_limit[k];
    } else {
        // symbols of lane l: positions kStep*t + 8*l + i < nc
        const int full_steps = nc / kStep, rem = nc % kStep;
        const int steps = (nc + kStep - 1) / kStep;
        int S[LPT];
#pragma unroll
        for (int k = 0; k < LPT; k++) S[k] = 8 * full_steps + max(0, min(8, rem - 8 * (lane + kLanes * k)));
        for (int tb = 0; tb < steps; tb += kEmitBlock) {
            const int te = min(tb + kEmitBlock, steps);
#pragma unroll
            for (int k = 0; k < LPT; k++) {
                const int full_runs = S[k] >> 3, tail = S[k] & 7;
                const int tf = min(te, full_runs);
                while (ld[k].runs() < tf) {
                    ld[k].step(pk, SLOW && refill_each, s.slim, s.soffs, s.ssyms, d.max_len, status);
                    ld[k].step(pk, true, s.slim, s.soffs, s.ssyms, d.max_len, status);
                }
                // a partial last run: its slot holds the codes after every lookup
                if (tail && full_runs < te)
                    while (ld[k].runs() == full_runs && ((ld[k].C >> kPbShift) & 0xFFu) < tail * BITS)
                        ld[k].step(pk, true, s.slim, s.soffs, s.ssyms, d.max_len, status);
            }
            __syncwarp();
            emit_ragged<BITS, OUT, LANES>(g, s, ost, first, nc, tb, te);
            __syncwarp();
        }
#pragma unroll
        for (int k = 0; k < LPT; k++)
            if (S[k] > 0) ok = ok && ld[k].bufa <= read_limit[k];
    }
    if (!ok) set_status(status, ENTRO_E_OVERRUN);
    __syncwarp();
}

__device__ __forceinline__ const GroupEntry &entry_at(const LaunchArgs &a, int i) {
    return a.table ? a.table[i] : a.one;
}

__device__ __forceinline__ bool chunk_words_ok(const DevTensor &d, long long c, int stage_rows, int lanes) {
    const uint64_t st = d.index[2 * c], nx = d.index[2 * c + 2];
    return nx >= st && nx <= static_cast<uint64_t>(d.payload_words) && (nx - st) % lanes == 0 &&
           (nx - st) / lanes + kSlackRows <= static_cast<uint64_t>(stage_rows);
}

// Issue the staging copy of a chunk whose words are [st, nx) (one lane).  An
// inconsistent index arrives with no bytes; the consumer re-checks and skips.
// A chunk's words [st, nx) into a staging buffer of stage_rows rows of `lanes`
// words; unit: the chunk sizes the format allows are multiples of it (lanes
// for word-interleaved lanes, 4 for consumption order).  A chunk that does not
// fit is not copied (the barrier completes with no bytes; the decode checks
// the same bounds and reports it).
__device__ __forceinline__ void issue_words(const DevTensor &d, uint64_t st, uint64_t nx, uint32_t *buf,
                                            uint64_t *bar, int stage_rows, int lanes, int unit) {
    const bool ok = nx >= st && nx <= static_cast<uint64_t>(d.payload_words) && (nx - st) % unit == 0 &&
                    (nx - st + lanes - 1) / lanes + kSlackRows <= static_cast<uint64_t>(stage_rows);
    const uint32_t bytes = ok ? static_cast<uint32_t>((nx - st) * 4) : 0u;
    mbar_arrive_expect_tx(bar, bytes);
    if (bytes) bulk_copy_g2s(buf, d.payload + st, bytes, bar);
}

__device__ __forceinline__ void issue_chunk(const DevTensor &d, long long c, uint32_t *buf, uint64_t *bar,
                                            int stage_rows, int lanes, int unit) {
    issue_words(d, d.index[2 * c], d.index[2 * c + 2], buf, bar, stage_rows, lanes, unit);
}

template <int BITS, int OUT, bool SLOW, int BPAD, int LANES>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) lanes_kernel(const __grid_constant__ LaunchArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int warps = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Smem s = carve(smem_raw, warps, a.x_elems, a.stage_rows * LANES, a.out_words, 0, kWideLutBytes);
    const Pipes pk{a.k_one, a.k_one << 2, a.k_one << 3, a.k_one << 8, a.k_one << 12, a.k_one << 24};
    uint64_t *bar = s.bars + 2 * warp;
    const size_t buf_words = static_cast<size_t>(a.stage_rows) * LANES;
    uint32_t *stage = s.stage + static_cast<size_t>(warp) * 2 * buf_words;
    uint32_t *ost = s.ostage + static_cast<size_t>(warp) * a.out_words;
    if (lane == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 1, 1);
    }
    if (threadIdx.x == 0) mbar_init(s.tbar, 1);
    fence_mbar_init();
    grid_launch_dependents();
    __syncthreads();

    // this CTA's share: chunks that start inside its symbol range
    const long long s0 = a.total_syms * blockIdx.x / gridDim.x;
    const long long s1 = a.total_syms * (blockIdx.x + 1) / gridDim.x;
    int ei = 0;
    {
        int lo = 0, hi = a.count - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (entry_at(a, mid).sym_begin <= s0) lo = mid;
            else hi = mid - 1;
        }
        ei = lo;
    }
    uint32_t phase0 = 0, phase1 = 0;  // completed phases of the two staging buffers
    uint32_t tphase = 0;              // completed phases of the table barrier
    bool dead = false;                // this warp gave up on a copy: it only keeps the CTA's barriers
    for (; ei < a.count; ei++) {
        const GroupEntry &g = entry_at(a, ei);
        if (g.sym_begin >= s1) break;
        const long long C = g.d.chunk_symbols;
        long long ca = s0 > g.sym_begin ? (s0 - g.sym_begin + C - 1) / C : 0;
        long long cb = (s1 - g.sym_begin + C - 1) / C;
        if (cb > g.d.n_chunks) cb = g.d.n_chunks;
        if (ca >= cb) continue;
        issue_tables<OUT, SLOW>(g, s, 2, a.batch, a.x_in_smem, a.tx_extra);
        // warp w takes chunks ca + w, ca + w + warps, ...  double buffered.  The
        // index entries of the first two are read by four lanes at once, and
        // both copies fly while the tables arrive.
        long long c = ca + warp;
        bool pend0 = false, pend1 = false;
        if (!dead) {
            const long long cq = (lane < 2) ? c : c + warps;
            uint64_t iv = 0;
            if (lane < 4 && cq < cb) iv = g.d.index[2 * cq + 2 * (lane & 1)];
            const uint64_t st0 = __shfl_sync(0xffffffffu, iv, 0), nx0 = __shfl_sync(0xffffffffu, iv, 1);
            const uint64_t st1 = __shfl_sync(0xffffffffu, iv, 2), nx1 = __shfl_sync(0xffffffffu, iv, 3);
            if (lane == 0) {
                if (c < cb) issue_words(g.d, st0, nx0, stage, bar, a.stage_rows, LANES, LANES);
                if (c + warps < cb)
                    issue_words(g.d, st1, nx1, stage + buf_words, bar + 1, a.stage_rows, LANES, LANES);
            }
            pend0 = c < cb;
            pend1 = c + warps < cb;
        }
        grid_wait_prior();
        issue_x<OUT>(g, s, a.batch, a.x_in_smem);
        const bool tables_ok = finish_tables<OUT, SLOW>(g, s, tphase);
        tphase++;
        if (!tables_ok) {
            // the table barrier may never complete: give up on every later entry, let this
            // entry's copies land (bounded waits) and leave
            set_status(a.status, ENTRO_E_TIMEOUT);
            if (pend0) mbar_wait(bar, phase0 & 1);
            if (pend1) mbar_wait(bar + 1, phase1 & 1);
            if (threadIdx.x == 0) mbar_wait(s.tbar, (tphase - 1) & 1);
            __syncthreads();
            return;
        }
        if (!dead) {
            for (int k = 0; c < cb; c += warps, k++) {
                const int b = k & 1;
                const uint32_t phase = b ? phase1 : phase0;
                const bool ok_wait = __all_sync(0xffffffffu, mbar_wait(bar + b, phase & 1));
                if (!ok_wait) {
                    set_status(a.status, ENTRO_E_TIMEOUT);
                    dead = true;
                    break;
                }
                if (b) { phase1++; pend1 = false; }
                else { phase0++; pend0 = false; }
                if (chunk_words_ok(g.d, c, a.stage_rows, LANES))
                    decode_chunk<BITS, OUT, SLOW, BPAD, LANES>(g, s, pk, stage + b * buf_words, ost, a.stage_rows,
                                                               c, a.batch, a.x_in_smem, a.status);
                else
                    set_status(a.status, ENTRO_E_CORRUPT);
                if (c + 2 * warps < cb) {
                    if (lane == 0) {
                        fence_proxy_async();
                        issue_chunk(g.d, c + 2 * warps, stage + b * buf_words, bar + b, a.stage_rows, LANES, LANES);
                    }
                    if (b) pend1 = true;
                    else pend0 = true;
                }
            }
        }
        if (dead) {
            // let copies still in flight land (bounded) before shared memory is reused
            if (pend0) mbar_wait(bar, phase0 & 1);
            if (pend1) mbar_wait(bar + 1, phase1 & 1);
        }
        __syncthreads();  // every warp done with this entry's tables
    }
}

// ------------------------------------------------------------------ batched GEMV on the tensor cores
//
// From batch 3 on, 3 to 16 products per decoded weight made the CUDA-core GEMV
// the bottleneck, and every warp streamed its own columns of x from L2.  This
// kernel decodes the same codes the same way, but the warps of a CTA work in
// lockstep on consecutive chunks (= consecutive rows, since its tensors have
// whole-row chunks) and multiply with mma.sync m16n8k16 (bf16 operands, fp32
// accumulation):
//   A = W[the CTA's 16 rows, 16 columns]                from the warps' run rings
//   B = x^T[16 columns, 8 batch rows] (1 or 2 tiles)    from global memory (L2)
//   D = y partials [16 rows, 8 batch rows]              registers, per warp
// Each lockstep block covers E runs of every chunk (E divides the runs of a
// row; E plus the runs a lane may complete after its last check fit the
// ring); after a CTA barrier the block's columns are split among the warps in
// groups of 32 (4 format lanes x 8 weights).  The k order inside an MMA is
// permuted so that each thread's A registers are the 8 weights of one ring
// slot and its B registers one 16-byte load of x:
//   k-step 0: k = 2j + e <-> column 8j + e, k = 2j + 8 + e <-> column 8j + 2 + e
//   k-step 1: the same with columns 8j + 4 + e and 8j + 6 + e  (j = lane % 4)
// The partial sums of a row are added across warps in warp order at the row's
// end (fixed order: the result does not depend on timing).  For a batch of up
// to 8 one MMA covers 256 weights.

constexpr int kTileMaxBlock = kRing - runs_per_check(kTileLookupsPerCheck);  // a block plus the slots a lane may write past it fit the ring
constexpr int kTileBatch = 4;             // padded batch from which the tensor-core GEMV runs

// Runs per lockstep block: the largest divisor of the runs per row that fits the ring.
__host__ __device__ inline int tile_block_runs(long long cols, int lanes) {
    const long long spr = cols / (kRun * lanes);
    for (int e = kTileMaxBlock; e > 1; e--)
        if (spr % e == 0) return e;
    return 1;
}

// Ring words per warp for the tensor-core GEMV: the ring plus a pad of `bits`
// words, which puts the rings of consecutive warps 4 (4-bit) or 8 (8-bit)
// banks apart, so the B-fragment loads of 8 rows hit 32 different banks (per
// half warp for the 8-byte loads of 8-bit codes).
__host__ __device__ inline int tile_ring_words(int bits, int lanes) { return kRing * lanes * bits / 4 + bits; }

__device__ __forceinline__ void mma_16816_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int BITS, bool SLOW, int LANES, int NB>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) gemv_mma_kernel(const __grid_constant__ LaunchArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    constexpr int LPT = LANES / kLanes;
    constexpr int kGroupsPerRun = LANES / 4;  // 32-column groups in one run step of a chunk
    const int warps = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;  // MMA fragment coordinates
    const Smem s = carve(smem_raw, warps, 0, a.stage_rows * LANES, a.out_words, static_cast<size_t>(warps) * NB * 32 * 16);
    uint64_t *bar = s.bars + 2 * warp;
    const size_t buf_words = static_cast<size_t>(a.stage_rows) * LANES;
    uint32_t *stage = s.stage + static_cast<size_t>(warp) * 2 * buf_words;
    uint32_t *ost = s.ostage + static_cast<size_t>(warp) * a.out_words;
    if (lane == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 1, 1);
    }
    if (threadIdx.x == 0) mbar_init(s.tbar, 1);
    fence_mbar_init();
    grid_launch_dependents();
    __syncthreads();

    const long long s0 = a.total_syms * blockIdx.x / gridDim.x;
    const long long s1 = a.total_syms * (blockIdx.x + 1) / gridDim.x;
    int ei = 0;
    {
        int lo = 0, hi = a.count - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (entry_at(a, mid).sym_begin <= s0) lo = mid;
            else hi = mid - 1;
        }
        ei = lo;
    }
    const int batch = a.batch;
    uint32_t phase0 = 0, phase1 = 0, tphase = 0;
    bool dead = false;  // this warp gave up on a copy: it decodes nothing more but keeps every barrier
    for (; ei < a.count; ei++) {
        const GroupEntry &g = entry_at(a, ei);
        if (g.sym_begin >= s1) break;
        const DevTensor &d = g.d;
        const long long C = d.chunk_symbols;
        long long ca = s0 > g.sym_begin ? (s0 - g.sym_begin + C - 1) / C : 0;
        long long cb = (s1 - g.sym_begin + C - 1) / C;
        if (cb > d.n_chunks) cb = d.n_chunks;
        if (ca >= cb) continue;
        issue_tables<OUT_GEMV, SLOW>(g, s, 1, batch, 0, a.tx_extra);
        bool pend0 = false, pend1 = false;
        if (!dead) {
            const long long c = ca + warp;
            const long long cq = (lane < 2) ? c : c + warps;
            uint64_t iv = 0;
            if (lane < 4 && cq < cb) iv = d.index[2 * cq + 2 * (lane & 1)];
            const uint64_t st0 = __shfl_sync(0xffffffffu, iv, 0), nx0 = __shfl_sync(0xffffffffu, iv, 1);
            const uint64_t st1 = __shfl_sync(0xffffffffu, iv, 2), nx1 = __shfl_sync(0xffffffffu, iv, 3);
            if (lane == 0) {
                if (c < cb) issue_words(d, st0, nx0, stage, bar, a.stage_rows, LANES, LANES);
                if (c + warps < cb) issue_words(d, st1, nx1, stage + buf_words, bar + 1, a.stage_rows, LANES, LANES);
            }
            pend0 = c < cb;
            pend1 = c + warps < cb;
        }
        grid_wait_prior();
        const bool tables_ok = finish_tables<OUT_GEMV, SLOW>(g, s, tphase);
        tphase++;
        if (!tables_ok) {
            set_status(a.status, ENTRO_E_TIMEOUT);
            if (pend0) mbar_wait(bar, phase0 & 1);
            if (pend1) mbar_wait(bar + 1, phase1 & 1);
            if (threadIdx.x == 0) mbar_wait(s.tbar, (tphase - 1) & 1);
            __syncthreads();
            return;
        }
        const int K = static_cast<int>(d.cols);
        const int spr = K / (kRun * LANES);                      // runs per row
        const int E = tile_block_runs(K, LANES);
        const int runs = static_cast<int>(C / (kRun * LANES));  // runs per chunk (whole rows)
        const int rows_per_chunk = static_cast<int>(C / K);
        const int groups = E * kGroupsPerRun;
        const bool refill_each = SLOW && d.max_len > 16;
        const uint4 *xg = reinterpret_cast<const uint4 *>(g.x);
        const int xrow = K >> 3;  // uint4 per row of x
        int k = 0;
        for (long long c0 = ca; c0 < cb; c0 += warps, k++) {
            const long long c = c0 + warp;
            const int nrows = static_cast<int>(cb - c0 < warps ? cb - c0 : warps);  // chunks (rows of W) in this group
            // a short last chunk holds whole rows, hence whole runs: it stops decoding early and its
            // missing rows are not written
            const int my_runs = c == d.n_chunks - 1 ? static_cast<int>((d.n - c * C) / (kRun * LANES)) : runs;
            const int b = k & 1;
            bool active = c < cb && !dead;
            if (active) {
                const uint32_t phase = b ? phase1 : phase0;
                if (!__all_sync(0xffffffffu, mbar_wait(bar + b, phase & 1))) {
                    set_status(a.status, ENTRO_E_TIMEOUT);
                    dead = true;
                    active = false;
                } else {
                    if (b) { phase1++; pend1 = false; }
                    else { phase0++; pend0 = false; }
                    if (!chunk_words_ok(d, c, a.stage_rows, LANES)) {
                        set_status(a.status, ENTRO_E_CORRUPT);
                        active = false;
                    }
                }
            }
            const uint32_t *buf = stage + b * buf_words;
            LaneDecoder<BITS, SLOW, LANES> ld[LPT];
            uint32_t read_limit[LPT];
            if (active) {
                const int words = static_cast<int>((d.index[2 * c + 2] - d.index[2 * c]) / LANES);
#pragma unroll
                for (int q = 0; q < LPT; q++) {
                    const int l = lane + kLanes * q;
                    ld[q].init(s, buf + l, ost + (BITS == 4 ? l : 2 * l), a.stage_rows - 1);
                    read_limit[q] = smem_addr(buf + l) + 4u * LANES * static_cast<uint32_t>(words + kOverrunRows);
                }
            }
            float acc[NB][4];
#pragma unroll
            for (int nb = 0; nb < NB; nb++)
#pragma unroll
                for (int i = 0; i < 4; i++) acc[nb][i] = 0.f;
            for (int tb = 0; tb < runs; tb += E) {
                const int te = tb + E;
                if (active && tb < my_runs) decode_to<kTileLookupsPerCheck>(ld, s, te, te, d.max_len, refill_each, a.status);
                const int col0 = (tb % spr) * (kRun * LANES);
                // The warp's groups q = warp, warp + warps, ... two per pass; the x
                // fragments of the first pass are loaded (from L2) before the
                // barrier, those of the next pass while this pass multiplies.
                // A = rows gid and gid + 8 of the group (the code rings of those
                // warps), B = x^T of batch rows 8 nb + gid.
                const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
                const uint32_t *ring_lo = s.ostage + static_cast<size_t>(gid) * a.out_words;
                const uint32_t *ring_hi = s.ostage + static_cast<size_t>(gid + 8) * a.out_words;
                const bool has_lo = gid < nrows, has_hi = gid + 8 < nrows;
                auto xload = [&](int q, uint4(&xr)[NB]) {
                    const int xo = ((col0 + 32 * q) >> 3) + tig;
#pragma unroll
                    for (int nb = 0; nb < NB; nb++) {
                        const int bb = 8 * nb + gid;
                        xr[nb] = q < groups && bb < batch ? __ldg(xg + bb * xrow + xo) : z4;
                    }
                };
                uint4 xc[2][NB];
                xload(warp, xc[0]);
                xload(warp + warps, xc[1]);
                __syncthreads();  // the block's runs of every row are in the rings
                for (int q0 = warp; q0 < groups; q0 += 2 * warps) {
                    uint4 xn[2][NB];
                    xload(q0 + 2 * warps, xn[0]);
                    xload(q0 + 3 * warps, xn[1]);
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const int q = q0 + h * warps;
                        if (q >= groups) break;
                        const int t = tb + q / kGroupsPerRun;
                        const int slot = LANES * (t & (kRing - 1)) + 4 * (q % kGroupsPerRun) + tig;
                        const uint4 wlo = has_lo ? values8<BITS>(s, ring_lo, slot) : z4;
                        const uint4 whi = has_hi ? values8<BITS>(s, ring_hi, slot) : z4;
#pragma unroll
                        for (int nb = 0; nb < NB; nb++) {
                            mma_16816_bf16(acc[nb], wlo.x, whi.x, wlo.y, whi.y, xc[h][nb].x, xc[h][nb].y);
                            mma_16816_bf16(acc[nb], wlo.z, whi.z, wlo.w, whi.w, xc[h][nb].z, xc[h][nb].w);
                        }
                    }
#pragma unroll
                    for (int h = 0; h < 2; h++)
#pragma unroll
                        for (int nb = 0; nb < NB; nb++) xc[h][nb] = xn[h][nb];
                }
                if (te % spr == 0) {
                    // row end: partial sums of every warp, added in warp order.  Thread
                    // 4 (r % 8) + n / 2 holds D[r][n] (element 2 (r >= 8) + n % 2).
                    float4 *rd = reinterpret_cast<float4 *>(s.red);
#pragma unroll
                    for (int nb = 0; nb < NB; nb++)
                        rd[(NB * warp + nb) * 32 + lane] = make_float4(acc[nb][0], acc[nb][1], acc[nb][2], acc[nb][3]);
                    __syncthreads();
                    const long long row_in_chunk = tb / spr;
                    for (int o = threadIdx.x; o < 256; o += blockDim.x) {
                        const int bb = o >> 4, r = o & 15;
                        const long long row = (c0 + r) * rows_per_chunk + row_in_chunk;
                        if (bb < batch && r < nrows && row < d.rows) {
                            const int nb = bb >> 3, n = bb & 7;
                            const int src = ((4 * (r & 7) + (n >> 1)) << 2) + ((r >> 3) << 1) + (n & 1);
                            float v = 0.f;
                            for (int w = 0; w < warps; w++) v += s.red[(NB * w + nb) * 128 + src];
                            g.y[static_cast<long long>(bb) * d.rows + row] = v;
                        }
                    }
#pragma unroll
                    for (int nb = 0; nb < NB; nb++)
#pragma unroll
                        for (int i = 0; i < 4; i++) acc[nb][i] = 0.f;
                }
                __syncthreads();  // every warp is done reading the rings before they are rewritten
            }
            if (active) {
                bool ok = true;
#pragma unroll
                for (int q = 0; q < LPT; q++) ok = ok && ld[q].bufa <= read_limit[q];
                if (!ok) set_status(a.status, ENTRO_E_OVERRUN);
            }
            if (c < cb && !dead && c + 2 * warps < cb) {
                if (lane == 0) {
                    fence_proxy_async();
                    issue_chunk(d, c + 2 * warps, stage + b * buf_words, bar + b, a.stage_rows, LANES, LANES);
                }
                if (b) pend1 = true;
                else pend0 = true;
            }
        }
        if (dead) {
            if (pend0) mbar_wait(bar, phase0 & 1);
            if (pend1) mbar_wait(bar + 1, phase1 & 1);
        }
        __syncthreads();
    }
}

#include "rows.cuh"

// ------------------------------------------------------------------ single-stream format
//
// One warp per chunk of the one-bitstream format (EntroLLM technical summary:
// the coded chunks decode in parallel).  The chunk's bits [B0, B1) are cut
// into 32 equal segments.  Lane i decodes from the start of segment i until it
// crosses into segment i+1 and notes where it stopped and how many codes it
// read.  Lane 0 starts on a code boundary; a lane whose start differs from
// where its left neighbour stopped decodes again from there, until no start
// changes (at most 32 rounds; Huffman codes resynchronise within a few codes,
// so two rounds are typical).  An exclusive warp-shuffle scan of the counts
// then gives every lane its first output position, and a last pass writes the
// codes or their bf16 values.

struct BitReader {
    const uint32_t *words;
    long long limit;  // readable words (payload + pad)
    long long k;      // next word to load
    uint64_t win;
    int nb;

    __device__ __forceinline__ uint32_t word(long long i) const { return i < limit ? __ldg(words + i) : 0u; }
    __device__ __forceinline__ void seek(uint64_t pos) {
        k = static_cast<long long>(pos >> 5);
        const int sh = static_cast<int>(pos & 31);
        win = ((static_cast<uint64_t>(word(k)) << 32) | word(k + 1)) << sh;
        nb = 64 - sh;
        k += 2;
    }
    __device__ __forceinline__ void refill() {
        if (nb <= 32) {
            win |= static_cast<uint64_t>(word(k)) << (32 - nb);
            nb += 32;
            k++;
        }
    }
    // one code; returns its table entry (length | symbol << 8)
    template <bool SLOW>
    __device__ __forceinline__ uint32_t next(const Smem &s, int max_len, int32_t *status) {
        refill();
        uint32_t e = s.lut[static_cast<uint32_t>(win >> (64 - kMaxLutBits))];
        if (SLOW && (e & 31u) == 0) e = slow_entry(win, max_len, s.slim, s.soffs, s.ssyms, status);
        const uint32_t len = e & 31u;
        win <<= len;
        nb -= static_cast<int>(len);
        return e;
    }
};

// Decode from bit `pos` (a code boundary) until crossing `stop`; returns the
// stop position and the number of codes read.
template <bool SLOW>
__device__ __forceinline__ uint64_t scan_segment(BitReader &br, const Smem &s, int max_len, uint64_t pos,
                                                 uint64_t stop, int max_codes, int *count, int32_t *status) {
    int n = 0;
    if (pos < stop) {
        br.seek(pos);
        while (pos < stop && n < max_codes) {
            pos += br.next<SLOW>(s, max_len, status) & 31u;
            n++;
        }
    }
    *count = n;
    return pos;
}

template <int BITS, int OUT, bool SLOW>
__global__ void __launch_bounds__(256) single_kernel(const __grid_constant__ LaunchArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const Smem s = carve(smem_raw, 0, 0, 0, 0);
    const GroupEntry &g = a.one;
    const DevTensor &d = g.d;
    if (threadIdx.x == 0) mbar_init(s.tbar, 1);
    fence_mbar_init();
    grid_launch_dependents();
    __syncthreads();
    issue_tables<OUT, SLOW>(g, s, 0, 1, 0, a.tx_extra);
    grid_wait_prior();
    if (!finish_tables<OUT, SLOW>(g, s, 0)) {
        set_status(a.status, ENTRO_E_TIMEOUT);
        if (threadIdx.x == 0) mbar_wait(s.tbar, 0);  // bounded: let the table copy land before leaving
        __syncthreads();
        return;
    }
    const int lane = threadIdx.x & 31;
    const long long c = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (c >= d.n_chunks) return;
    const uint64_t B0 = d.index[2 * c], B1 = d.index[2 * c + 2];
    const long long first = static_cast<long long>(d.index[2 * c + 1]);
    const long long nc = static_cast<long long>(d.index[2 * c + 3]) - first;
    if (B1 < B0 || (B1 + 31) / 32 > static_cast<uint64_t>(d.payload_words) || nc < 0 || nc > d.chunk_symbols) {
        if (lane == 0) set_status(a.status, ENTRO_E_CORRUPT);
        return;
    }
    BitReader br{d.payload, d.payload_words + kPadWords, 0, 0, 0};
    const uint64_t L = B1 - B0;
    const uint64_t seg0 = B0 + L * lane / 32, seg1 = (lane == 31) ? B1 : B0 + L * (lane + 1) / 32;
    // every code takes at least one bit: a segment never holds more codes than bits
    const int cap = static_cast<int>(min(static_cast<long long>(seg1 - seg0) + 64, nc + 1));
    uint64_t start = seg0;
    int n = 0;
    uint64_t end = scan_segment<SLOW>(br, s, d.max_len, start, seg1, cap, &n, a.status);
    for (int round = 0; round < 32; round++) {
        uint64_t prev = __shfl_up_sync(0xffffffffu, end, 1);
        if (lane == 0) prev = B0;
        const bool redo = prev != start;
        if (!__any_sync(0xffffffffu, redo)) break;
        if (redo) {
            start = prev;
            end = scan_segment<SLOW>(br, s, d.max_len, start, seg1, cap, &n, a.status);
        }
    }
    // output position of this lane's first code: exclusive scan of the counts
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    const uint64_t last_end = __shfl_sync(0xffffffffu, end, 31);
    if (total != nc || last_end != B1) {
        if (lane == 0) set_status(a.status, ENTRO_E_CORRUPT);
        return;
    }
    long long p = first + (incl - n);
    if (n > 0) br.seek(start);
    uint8_t *o8 = reinterpret_cast<uint8_t *>(g.out);
    uint16_t *o16 = reinterpret_cast<uint16_t *>(g.out);
    // 4-bit codes: chunks start on even symbols (checked on the host), so only
    // a lane's first and last codes can share a byte with a neighbour lane;
    // those nibbles go through a word-wide atomic, the rest as whole bytes.
    uint32_t pending = 0;
    for (int i = 0; i < n; i++, p++) {
        const uint32_t sym = (br.next<SLOW>(s, d.max_len, a.status) >> 8) & 0xFFu;
        if (OUT == OUT_BF16) {
            o16[p] = static_cast<uint16_t>(s.vtab[sym]);
        } else if (BITS == 8) {
            o8[p] = static_cast<uint8_t>(sym);
        } else {
            const bool lo_half = (p & 1) == 0;
            const bool shared_byte = (lo_half && i == n - 1 && p + 1 < first + nc) || (!lo_half && i == 0);
            if (shared_byte) {
                uint32_t *word = reinterpret_cast<uint32_t *>(o8 + ((p >> 1) & ~3LL));
                const int shift = static_cast<int>(((p >> 1) & 3) * 8 + (lo_half ? 0 : 4));
                atomicAnd(word, ~(0xFu << shift));
                atomicOr(word, sym << shift);
            } else if (lo_half) {
                pending = sym;
                if (p + 1 == first + nc) o8[p >> 1] = static_cast<uint8_t>(pending);
            } else {
                o8[p >> 1] = static_cast<uint8_t>(pending | (sym << 4));
            }
        }
    }
}

// ------------------------------------------------------------------ single-stream format, CTA per chunk
//
// For chunks of up to kSegChunkSymbols codes: one CTA of kSegThreads threads
// per chunk, the chunk's words staged in shared memory by one bulk copy.  The
// chunk's bits [B0, B1) are cut into kSegThreads segments whose inner bounds
// are multiples of 32 bits.
//   1. Thread i decodes from the start of its segment until it crosses the
//      end and marks, in a bitmap of the chunk's bits, where each of its codes
//      began.  (Thread 0 starts on a code boundary; the others usually not.)
//   2. A thread whose start differs from where its left neighbour stopped
//      decodes again from there, but only until it reaches a position it
//      marked: from a common code boundary the two decodings are the same, so
//      the rest of its codes are the marked ones (a popcount) and its end
//      stands.  Rounds repeat until no start changes; Huffman codes
//      resynchronise within a few codes, so one round of a few codes is usual.
//   3. A block-wide exclusive scan of the counts places every thread's codes;
//      each thread decodes them once more into a shared-memory copy of the
//      chunk's output, which the CTA writes out with coalesced stores.

constexpr int kSegThreads = 256;
constexpr int kSegChunkSymbols = 16384;

struct SegLayout {
    size_t words, bitmap, out, ends, counts, wsum, total;
};

// stage_words: staged words per chunk (a multiple of 4)
__host__ __device__ inline SegLayout seg_layout(int stage_words, int chunk_symbols) {
    SegLayout o;
    size_t p = align_up(smem_layout(0, 0, 0, 0).total, 16);
    o.words = p;
    p += (size_t)stage_words * 4;
    o.bitmap = p;
    p += (size_t)stage_words * 4;
    o.out = p;
    p = align_up(p + (size_t)chunk_symbols, 16);
    o.ends = p;
    p += kSegThreads * 8;
    o.counts = p;
    p += kSegThreads * 4;
    o.wsum = p;
    p += (kSegThreads / 32) * 4;
    o.total = align_up(p, 16);
    return o;
}

struct SegReader {
    uint32_t base;    // shared address of staged word 0
    uint64_t bit0;    // stream position of staged word 0
    uint32_t k;       // next staged word
    uint32_t hi, lo;  // 64-bit window, MSB first
    int nb;           // valid bits in the window

    __device__ __forceinline__ uint32_t word(uint32_t i) const { return lds32(base + 4u * i); }
    __device__ __forceinline__ void seek(uint64_t pos) {
        const uint32_t rel = static_cast<uint32_t>(pos - bit0);
        k = rel >> 5;
        const uint32_t sh = rel & 31;
        const uint32_t w0 = word(k), w1 = word(k + 1);
        hi = __funnelshift_l(w1, w0, sh);
        lo = w1 << sh;
        nb = 64 - static_cast<int>(sh);
        k += 2;
    }
    // one code; returns its table entry (length | symbol << 8)
    template <bool SLOW>
    __device__ __forceinline__ uint32_t next(const Smem &s, int max_len, int32_t *status) {
        // branch-free refill: word k is always in the staged range (4 words of slack)
        const bool need = nb <= 32;
        const uint32_t wv = need ? word(k) : 0u, n = static_cast<uint32_t>(nb);
        hi |= shr_clamp(wv, n);
        lo |= shl_clamp(wv, 32u - n);
        nb += need ? 32 : 0;
        k += need ? 1u : 0u;
        uint32_t e = lds32(smem_addr(s.lut) + ((hi >> (32 - kMaxLutBits)) << 2));
        if (SLOW && (e & 31u) == 0)
            e = slow_entry((static_cast<uint64_t>(hi) << 32) | lo, max_len, s.slim, s.soffs, s.ssyms, status);
        const uint32_t len = e & 31u;
        hi = __funnelshift_l(lo, hi, len);
        lo <<= len;
        nb -= static_cast<int>(len);
        return e;
    }
};

template <int BITS, int OUT, bool SLOW>
__global__ void __launch_bounds__(kSegThreads) segment_kernel(const __grid_constant__ LaunchArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const Smem s = carve(smem_raw, 0, 0, 0, 0);
    const SegLayout L = seg_layout(a.stage_rows, static_cast<int>(a.one.d.chunk_symbols));
    uint32_t *words = reinterpret_cast<uint32_t *>(smem_raw + L.words);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(smem_raw + L.bitmap);
    uint8_t *ostage = smem_raw + L.out;
    uint64_t *ends = reinterpret_cast<uint64_t *>(smem_raw + L.ends);
    int *counts = reinterpret_cast<int *>(smem_raw + L.counts);
    int *wsum = reinterpret_cast<int *>(smem_raw + L.wsum);
    const GroupEntry &g = a.one;
    const DevTensor &d = g.d;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long c = blockIdx.x;
    const uint64_t B0 = d.index[2 * c], B1 = d.index[2 * c + 2];
    const long long first = static_cast<long long>(d.index[2 * c + 1]);
    const long long nc = static_cast<long long>(d.index[2 * c + 3]) - first;
    const uint64_t w0 = (B0 >> 5) & ~3ull;                     // 16-byte aligned start of the copy
    const uint64_t w1 = (((B1 + 31) >> 5) + 4 + 3) & ~3ull;    // past the chunk's last word, 4 words of slack
    const bool sane = B1 >= B0 && (B1 + 31) / 32 <= static_cast<uint64_t>(d.payload_words) && nc >= 0 &&
                      nc <= d.chunk_symbols && w1 - w0 <= static_cast<uint64_t>(a.stage_rows);
    if (tid == 0) mbar_init(s.tbar, 1);
    fence_mbar_init();
    grid_launch_dependents();
    __syncthreads();
    if (tid == 0) {
        // tables and the chunk's words on one barrier
        const uint32_t wbytes = sane ? static_cast<uint32_t>((w1 - w0) * 4) : 0u;
        uint32_t bytes = kLutSize * 4 + wbytes + a.tx_extra;
        if (SLOW) bytes += kSlowBytes;
        mbar_arrive_expect_tx(s.tbar, bytes);
        bulk_copy_g2s(s.lut, d.lut, kLutSize * 4, s.tbar);
        if (SLOW) bulk_copy_g2s(s.slim, d.slow_limit, kSlowBytes, s.tbar);
        if (wbytes) bulk_copy_g2s(words, d.payload + w0, wbytes, s.tbar);
    }
    for (int i = tid; i < a.stage_rows; i += kSegThreads) bitmap[i] = 0u;
    grid_wait_prior();
    if (!finish_tables<OUT, SLOW>(g, s, 0)) {
        set_status(a.status, ENTRO_E_TIMEOUT);
        if (tid == 0) mbar_wait(s.tbar, 0);  // bounded: let the copies land before leaving
        __syncthreads();
        return;
    }
    if (!sane) {
        if (tid == 0) set_status(a.status, ENTRO_E_CORRUPT);
        return;
    }
    SegReader rd{smem_addr(words), w0 * 32, 0, 0, 0};
    const uint64_t span = B1 - B0;
    auto bound = [&](int i) -> uint64_t {
        if (i <= 0) return B0;
        if (i >= kSegThreads) return B1;
        const uint64_t b = (B0 + span * static_cast<uint64_t>(i) / kSegThreads + 31) & ~31ull;
        return b < B1 ? b : B1;
    };
    const uint64_t seg0 = bound(tid), seg1 = bound(tid + 1);
    // every code takes at least one bit: a segment never holds more codes than bits
    const int cap = static_cast<int>(min(static_cast<long long>(seg1 - seg0) + 64, nc + 1));

    // 1. scan from the segment start, marking code starts (bitmap words are this thread's own)
    int n1 = 0;
    uint64_t pos = seg0;
    if (seg0 < seg1) {
        rd.seek(seg0);
        // the current bitmap word is stored after every code (no branch)
        const uint32_t bm = smem_addr(bitmap);
        uint32_t bwi = 0xFFFFFFFFu, bw = 0u;
        while (pos < seg1 && n1 < cap) {
            const uint32_t rel = static_cast<uint32_t>(pos - rd.bit0);
            const uint32_t wi = rel >> 5;
            bw = (wi == bwi ? bw : 0u) | (0x80000000u >> (rel & 31));
            bwi = wi;
            sts32(bm + 4u * wi, bw);
            pos += rd.next<SLOW>(s, d.max_len, a.status) & 31u;
            n1++;
        }
    }
    const uint64_t end1 = pos;
    uint64_t start = seg0, end = end1;
    int n = n1;
    ends[tid] = end1;
    __syncthreads();

    // 2. resynchronise with the left neighbour
    bool bad = false;
    for (int round = 0; round < kSegThreads; round++) {
        const uint64_t prev = tid == 0 ? B0 : ends[tid - 1];
        const bool redo = prev != start;
        __syncthreads();
        if (redo) {
            start = prev;
            if (prev >= seg1) {
                n = 0;
                end = prev;
            } else {
                rd.seek(prev);
                uint64_t q = prev;
                int m = 0;
                for (;;) {
                    if (q >= seg1) {
                        n = m;
                        end = q;
                        break;
                    }
                    const uint32_t rel = static_cast<uint32_t>(q - rd.bit0);
                    if ((bitmap[rel >> 5] << (rel & 31)) & 0x80000000u) {
                        // a code this thread decoded in step 1 starts here: the rest is step 1's
                        const uint32_t last = static_cast<uint32_t>(seg1 - 1 - rd.bit0) >> 5;
                        int rest = __popc(bitmap[rel >> 5] & (0xFFFFFFFFu >> (rel & 31)));
                        for (uint32_t wi = (rel >> 5) + 1; wi <= last; wi++) rest += __popc(bitmap[wi]);
                        n = m + rest;
                        end = end1;
                        break;
                    }
                    if (m >= cap) {
                        bad = true;
                        n = 0;
                        end = q;
                        break;
                    }
                    q += rd.next<SLOW>(s, d.max_len, a.status) & 31u;
                    m++;
                }
            }
            ends[tid] = end;
        }
        if (!__syncthreads_or(redo)) break;
    }

    // 3. place: exclusive scan of the counts over the CTA
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    counts[tid] = n;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kSegThreads / 32; w++) {
        if (w < warp) before += wsum[w];
        total += wsum[w];
    }
    const int p0 = before + incl - n;
    if (__syncthreads_or(bad) || total != nc || ends[kSegThreads - 1] != B1) {
        if (tid == 0) set_status(a.status, ENTRO_E_CORRUPT);
        return;
    }
    if (n > 0) {
        rd.seek(start);
        for (int j = 0; j < n; j++) ostage[p0 + j] = static_cast<uint8_t>(rd.next<SLOW>(s, d.max_len, a.status) >> 8);
    }
    __syncthreads();
    const int ncodes = static_cast<int>(nc);
    if (OUT == OUT_BF16) {
        uint16_t *o16 = reinterpret_cast<uint16_t *>(g.out) + first;
        if ((first & 1) == 0) {
            uint32_t *o32 = reinterpret_cast<uint32_t *>(o16);
            for (int j = tid; 2 * j + 1 < ncodes; j += kSegThreads)
                o32[j] = (s.vtab[ostage[2 * j]] & 0xFFFFu) | (s.vtab[ostage[2 * j + 1]] << 16);
            if ((ncodes & 1) && tid == 0) o16[ncodes - 1] = static_cast<uint16_t>(s.vtab[ostage[ncodes - 1]]);
        } else {
            for (int j = tid; j < ncodes; j += kSegThreads) o16[j] = static_cast<uint16_t>(s.vtab[ostage[j]]);
        }
    } else if (BITS == 8) {
        uint8_t *o8 = reinterpret_cast<uint8_t *>(g.out) + first;
        if ((first & 15) == 0) {
            uint4 *o = reinterpret_cast<uint4 *>(o8);
            const uint4 *src = reinterpret_cast<const uint4 *>(ostage);
            for (int j = tid; j < ncodes / 16; j += kSegThreads) o[j] = src[j];
            for (int j = (ncodes & ~15) + tid; j < ncodes; j += kSegThreads) o8[j] = ostage[j];
        } else {
            for (int j = tid; j < ncodes; j += kSegThreads) o8[j] = ostage[j];
        }
    } else {
        // 4-bit: the chunk starts on an even code (checked on the host); code 2j in the low nibble
        uint8_t *o8 = reinterpret_cast<uint8_t *>(g.out) + (first >> 1);
        for (int j = tid; 2 * j < ncodes; j += kSegThreads) {
            const uint32_t hi = 2 * j + 1 < ncodes ? ostage[2 * j + 1] : 0u;
            o8[j] = static_cast<uint8_t>((ostage[2 * j] & 15u) | (hi << 4));
        }
    }
}

// ------------------------------------------------------------------ host side

// Message of the last CUDA runtime error the library saw on this host thread.
static thread_local char g_cuda_msg[160] = "";

static int cuda_fail(cudaError_t e, const char *where) {
    snprintf(g_cuda_msg, sizeof(g_cuda_msg), "%s: %s (%d)", where, cudaGetErrorString(e), (int)e);
    return ENTRO_E_CUDA;
}

struct DeviceInfo {
    int sms = 0;
    int smem_optin = 0;
};

static std::mutex g_mu;
constexpr int kMaxDevices = 64;
static DeviceInfo g_dev[kMaxDevices];

static int device_info(int dev, DeviceInfo *out) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev < 0 || dev >= kMaxDevices) return ENTRO_E_LIMIT;
    DeviceInfo &di = g_dev[dev];
    if (di.sms == 0) {
        cudaError_t e = cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&di.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) {
            di.sms = 0;
            return cuda_fail(e, "cudaDeviceGetAttribute");
        }
    }
    *out = di;
    return ENTRO_OK;
}

// Host-built decode tables of one tensor (canonical codes, RFC 1951 order).
//   lut:  12-bit peek -> (length, symbol) of the first code, 0 if longer than 12
//   mlut: 12-bit peek -> every whole code inside the 12 bits, up to 6 (4-bit)
//         or 3 (8-bit): bits used | count << 4 | symbols << 8
//   limit / offs / syms: canonical description for codes longer than 12 bits
//   wlut: 12-bit peek -> {every whole code inside the 12 bits, up to 8 (4-bit)
//         or 4 (8-bit), first code in the low bits; bits used | count * bits << 8}
static void build_tables(const uint8_t *len, int max_len, int bits, uint32_t *lut, uint32_t *mlut, uint32_t *wlut,
                         uint32_t *limit, int32_t *offs, uint8_t *syms, int *n_codes) {
    uint32_t code[256];
    canonical_codes(len, code);
    std::memset(lut, 0, kLutSize * 4);
    int count[33] = {0};
    int nz = 0;
    for (int s = 0; s < 256; s++) {
        if (!len[s]) continue;
        nz++;
        count[len[s]]++;
        if (len[s] <= kMaxLutBits) {
            const uint32_t lo = code[s] << (kMaxLutBits - len[s]);
            const uint32_t hi = (code[s] + 1) << (kMaxLutBits - len[s]);
            for (uint32_t i = lo; i < hi; i++) lut[i] = static_cast<uint32_t>(len[s]) | (static_cast<uint32_t>(s) << 8);
        }
    }
    *n_codes = nz;
    const int per = bits == 4 ? kMaxCodesPerLookup : kMaxCodesPerLookup / 2;
    for (uint32_t v = 0; v < (uint32_t)kLutSize; v++) {
        uint32_t used = 0, k = 0, packed = 0;
        while ((int)k < per) {
            const uint32_t e = lut[(v << used) & (kLutSize - 1)];
            const uint32_t l = e & 31u;
            if (l == 0 || used + l > (uint32_t)kMaxLutBits) break;
            packed |= ((e >> 8) & 0xFFu) << (bits * k);
            used += l;
            k++;
        }
        mlut[v] = used | (k << 4) | (packed << 8);
    }
    const int wide = wide_max_codes(bits);
    for (uint32_t v = 0; v < (uint32_t)kLutSize; v++) {
        uint32_t used = 0, k = 0, packed = 0;
        while ((int)k < wide) {
            const uint32_t e = lut[(v << used) & (kLutSize - 1)];
            const uint32_t l = e & 31u;
            if (l == 0 || used + l > (uint32_t)kMaxLutBits) break;
            packed |= ((e >> 8) & 0xFFu) << (bits * k);
            used += l;
            k++;
        }
        wlut[2 * v] = packed;
        wlut[2 * v + 1] = used | ((k * (uint32_t)bits) << kPbShift);
    }
    uint32_t first[33] = {0};
    int base[33] = {0};
    uint32_t c = 0;
    int rank = 0;
    for (int l = 1; l <= 32; l++) {
        c = (c + static_cast<uint32_t>(count[l - 1])) << 1;
        first[l] = c;
        base[l] = rank;
        rank += count[l];
    }
    for (int l = 0; l < 32; l++) {
        limit[l] = 0;
        offs[l] = 0;
        if (l >= 1 && l <= max_len) {
            limit[l] = (first[l] + static_cast<uint32_t>(count[l])) << (max_len - l);
            offs[l] = base[l] - static_cast<int32_t>(first[l]);
        }
    }
    int k = 0;
    std::memset(syms, 0, 256);
    for (int l = 1; l <= max_len; l++)
        for (int s = 0; s < 256; s++)
            if (len[s] == l) syms[k++] = static_cast<uint8_t>(s);
}

struct ImageLayout {
    uint64_t lut, mlut, wlut, slow, index, payload, total;
};

static ImageLayout image_layout(const Blob &b) {
    ImageLayout L;
    L.lut = 0;
    L.mlut = align256(L.lut + kLutSize * 4);
    L.wlut = align256(L.mlut + kLutSize * 4);
    L.slow = align256(L.wlut + kWideLutBytes);
    L.index = align256(L.slow + kSlowBytes);
    L.payload = align256(L.index + 16 * (b.header.n_chunks + 1));
    L.total = align256(L.payload + 4 * (b.header.payload_words + kPadWords));
    return L;
}

}  // namespace entro

using namespace entro;

extern "C" int entro_device_bytes(const entro_blob *blob, uint64_t *bytes) {
    if (!blob || !bytes) return ENTRO_E_INVAL;
    *bytes = image_layout(*reinterpret_cast<const Blob *>(blob)).total;
    return ENTRO_OK;
}

extern "C" int entro_upload(const entro_blob *blob, void *d_mem, uint64_t d_bytes, void *stream,
                            entro_tensor **out) {
    if (!blob || !out || !d_mem) return ENTRO_E_INVAL;
    *out = nullptr;
    const Blob &b = *reinterpret_cast<const Blob *>(blob);
    const ImageLayout L = image_layout(b);
    if (d_bytes < L.total || (reinterpret_cast<uintptr_t>(d_mem) & 255)) return ENTRO_E_INVAL;
    if (b.header.format != ENTRO_FORMAT_SINGLE && b.max_chunk_words > 16384) return ENTRO_E_LIMIT;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ENTRO_E_CUDA;
    TensorHandle *t = new (std::nothrow) TensorHandle();
    if (!t) return ENTRO_E_NOMEM;
    std::vector<uint8_t> host(L.index - L.lut, 0);
    uint32_t *lut = reinterpret_cast<uint32_t *>(host.data());
    uint32_t *mlut = reinterpret_cast<uint32_t *>(host.data() + L.mlut);
    uint32_t *wlut = reinterpret_cast<uint32_t *>(host.data() + L.wlut);
    uint32_t *limit = reinterpret_cast<uint32_t *>(host.data() + L.slow);
    int32_t *offs = reinterpret_cast<int32_t *>(host.data() + L.slow + 128);
    uint8_t *syms = host.data() + L.slow + 256;
    int n_codes = 0;
    build_tables(b.lengths, (int)b.header.max_len, (int)b.header.bits, lut, mlut, wlut, limit, offs, syms,
                 &n_codes);
    uint8_t *base = static_cast<uint8_t *>(d_mem);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint8_t *src = b.bytes.data();
    cudaError_t e = cudaMemcpyAsync(base, host.data(), host.size(), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(base + L.index, src + index_offset(), 16 * (b.header.n_chunks + 1),
                            cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess && b.header.payload_words)
        e = cudaMemcpyAsync(base + L.payload, src + payload_offset(b.header.n_chunks), 4 * b.header.payload_words,
                            cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(base + L.payload + 4 * b.header.payload_words, 0, 4 * kPadWords, st);
    // pageable sources: make sure the host staging above is consumed before `host` dies
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        delete t;
        return ENTRO_E_CUDA;
    }
    DevTensor &d = t->d;
    d.lut = reinterpret_cast<const uint32_t *>(base + L.lut);
    d.mlut = reinterpret_cast<const uint32_t *>(base + L.mlut);
    d.wlut = reinterpret_cast<const uint2 *>(base + L.wlut);
    d.slow_limit = reinterpret_cast<const uint32_t *>(base + L.slow);
    d.slow_offs = reinterpret_cast<const int32_t *>(base + L.slow + 128);
    d.slow_syms = base + L.slow + 256;
    d.index = reinterpret_cast<const uint64_t *>(base + L.index);
    d.payload = reinterpret_cast<const uint32_t *>(base + L.payload);
    d.n = (long long)b.header.n;
    d.rows = (long long)b.header.rows;
    d.cols = (long long)b.header.cols;
    d.chunk_symbols = (long long)b.header.chunk_symbols;
    d.n_chunks = (long long)b.header.n_chunks;
    d.payload_words = (long long)b.header.payload_words;
    std::memcpy(&d.scale, &b.header.scale_bits, 4);
    d.zero = b.header.zero;
    d.bits = (int)b.header.bits;
    d.max_len = (int)b.header.max_len;
    d.format = (int)b.header.format;
    d.max_chunk_words = (int)b.max_chunk_words;
    d.n_codes = n_codes;
    d.lanes = (int)b.header.lanes;
    t->device = dev;
    t->slow = d.max_len > kMaxLutBits || n_codes == 1;
    t->device_bytes = L.total;
    *out = reinterpret_cast<entro_tensor *>(t);
    return ENTRO_OK;
}

extern "C" void entro_tensor_free(entro_tensor *t) { delete reinterpret_cast<TensorHandle *>(t); }

namespace entro {

using LanesFn = void (*)(LaunchArgs);

template <int BITS, int OUT, bool SLOW, int LANES>
static LanesFn pick_bpad(int bpad) {
    if (OUT != OUT_GEMV) return lanes_kernel<BITS, OUT, SLOW, 1, LANES>;
    switch (bpad) {
        case 1: return lanes_kernel<BITS, OUT, SLOW, 1, LANES>;
        case 2: return lanes_kernel<BITS, OUT, SLOW, 2, LANES>;
        default: return nullptr;  // padded batch 4 to 16: gemv_mma_kernel
    }
}

template <int BITS, int LANES>
static LanesFn pick_out(int out, bool slow, int bpad) {
    if (out == OUT_CODES) return slow ? pick_bpad<BITS, OUT_CODES, true, LANES>(1) : pick_bpad<BITS, OUT_CODES, false, LANES>(1);
    if (out == OUT_BF16) return slow ? pick_bpad<BITS, OUT_BF16, true, LANES>(1) : pick_bpad<BITS, OUT_BF16, false, LANES>(1);
    return slow ? pick_bpad<BITS, OUT_GEMV, true, LANES>(bpad) : pick_bpad<BITS, OUT_GEMV, false, LANES>(bpad);
}

static LanesFn pick_lanes(int bits, int out, bool slow, int bpad, int lanes) {
    if (bits == 4) return lanes == 64 ? pick_out<4, 64>(out, slow, bpad) : pick_out<4, 32>(out, slow, bpad);
    return lanes == 64 ? pick_out<8, 64>(out, slow, bpad) : pick_out<8, 32>(out, slow, bpad);
}

template <int NB>
static LanesFn pick_mma_nb(int bits, bool slow, int lanes) {
    if (bits == 4) {
        if (lanes == 64) return slow ? gemv_mma_kernel<4, true, 64, NB> : gemv_mma_kernel<4, false, 64, NB>;
        return slow ? gemv_mma_kernel<4, true, 32, NB> : gemv_mma_kernel<4, false, 32, NB>;
    }
    if (lanes == 64) return slow ? gemv_mma_kernel<8, true, 64, NB> : gemv_mma_kernel<8, false, 64, NB>;
    return slow ? gemv_mma_kernel<8, true, 32, NB> : gemv_mma_kernel<8, false, 32, NB>;
}

// NB = 8-row tiles of the batch (B operand of the MMAs)
static int mma_batch_tiles(int batch) { return batch > 8 ? 2 : 1; }

static LanesFn pick_mma(int bits, bool slow, int lanes, int batch) {
    return mma_batch_tiles(batch) == 2 ? pick_mma_nb<2>(bits, slow, lanes) : pick_mma_nb<1>(bits, slow, lanes);
}

// The tensor-core GEMV needs chunks of whole rows (every GEMV tensor has them).
static bool mma_eligible(const DevTensor &d) {
    return d.cols > 0 && d.chunk_symbols % d.cols == 0;
}

static LanesFn pick_single(int bits, int out, bool slow) {
    if (bits == 4) {
        if (out == OUT_CODES) return slow ? single_kernel<4, OUT_CODES, true> : single_kernel<4, OUT_CODES, false>;
        return slow ? single_kernel<4, OUT_BF16, true> : single_kernel<4, OUT_BF16, false>;
    }
    if (out == OUT_CODES) return slow ? single_kernel<8, OUT_CODES, true> : single_kernel<8, OUT_CODES, false>;
    return slow ? single_kernel<8, OUT_BF16, true> : single_kernel<8, OUT_BF16, false>;
}

// Opt a kernel into `bytes` of dynamic shared memory and report how many CTAs
// of `threads` fit on one SM.  The opt-in attribute only ever grows (it is a
// per-kernel maximum, so a smaller later launch must not lower it below a
// larger cached one); occupancy is cached per (kernel, device, threads, bytes).
struct KernelConfig {
    const void *fn;
    int device, threads;
    size_t bytes;
    int per_sm;
};
struct KernelOptIn {
    const void *fn;
    int device;
    size_t bytes;
};
// Fixed-size caches: a launch never touches the host heap.
constexpr int kMaxConfigs = 512;
static KernelConfig g_kcfg[kMaxConfigs];
static int g_nkcfg = 0;
static KernelOptIn g_optin[kMaxConfigs];
static int g_noptin = 0;

static int kernel_config(const void *fn, int device, int threads, size_t bytes, int *per_sm) {
    std::lock_guard<std::mutex> lk(g_mu);
    KernelOptIn *opt = nullptr;
    for (int i = 0; i < g_noptin; i++)
        if (g_optin[i].fn == fn && g_optin[i].device == device) opt = &g_optin[i];
    if (!opt || opt->bytes < bytes) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        if (opt) opt->bytes = bytes;
        else if (g_noptin < kMaxConfigs) g_optin[g_noptin++] = {fn, device, bytes};
    }
    for (int i = 0; i < g_nkcfg; i++) {
        const KernelConfig &k = g_kcfg[i];
        if (k.fn == fn && k.device == device && k.threads == threads && k.bytes == bytes) {
            *per_sm = k.per_sm;
            return ENTRO_OK;
        }
    }
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (n < 1) {
        snprintf(g_cuda_msg, sizeof(g_cuda_msg), "no CTA of %d threads and %zu bytes fits an SM", threads, bytes);
        return ENTRO_E_CUDA;
    }
    if (g_nkcfg < kMaxConfigs) g_kcfg[g_nkcfg++] = {fn, device, threads, bytes, n};
    *per_sm = n;
    return ENTRO_OK;
}

// Launch overlap (programmatic dependent launch), off unless the caller turns it on.
static std::atomic<int> g_overlap{0};
// Bounded-wait test hook: bytes every launch adds to its table barrier that never arrive.
static std::atomic<uint32_t> g_tx_extra{0};

// overlap_ok: the kernel fills each SM with one CTA (the next launch's CTAs
// cannot move in before this one's leave).  Kernels with several CTAs per SM
// launch without overlap: the next launch's CTAs would become resident early
// and compete with the running ones (the 1024x1024 single-stream step was
// 44.5 us with overlap, 32.9 us without).
static cudaError_t launch(LanesFn fn, unsigned grid, unsigned threads, size_t smem, cudaStream_t st,
                          const LaunchArgs &a, bool overlap_ok = true) {
    if (!overlap_ok || !g_overlap.load(std::memory_order_relaxed)) {
        fn<<<grid, threads, smem, st>>>(a);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fn, a);
}

static int bpad_for(int batch) {
    int b = 1;
    while (b < batch) b <<= 1;
    return b;
}

static constexpr long long kXSmemElems = 48 * 1024;  // up to 96 KB of bf16 activations per CTA
static constexpr long long kXL1Bytes = 16 * 1024;    // activations that grouped launches read through L1

// Launch the lanes kernel over `count` entries (table on device, or `one`).
static int launch_lanes(const TensorHandle *const *ts, int count, int out_kind, int batch, const GroupEntry *d_table,
                        const GroupEntry &one, int32_t *status, cudaStream_t st) {
    bool slow = false;
    const int bits = ts[0]->d.bits, lanes = ts[0]->d.lanes;
    int max_words = 0;
    long long max_kb = 0, max_chunk = 0, total = 0;
    for (int i = 0; i < count; i++) {
        const DevTensor &d = ts[i]->d;
        if (d.bits != bits || d.lanes != lanes) return ENTRO_E_INVAL;
        slow = slow || ts[i]->slow;
        max_words = std::max(max_words, d.max_chunk_words);
        max_chunk = std::max(max_chunk, d.chunk_symbols);
        max_kb = std::max(max_kb, d.cols * (long long)bpad_for(batch));
        total += d.n;
    }
    if (total == 0) return ENTRO_OK;
    DeviceInfo di;
    if (device_info(ts[0]->device, &di) != ENTRO_OK) return ENTRO_E_CUDA;
    const int bpad = out_kind == OUT_GEMV ? bpad_for(batch) : 1;
    bool mma = out_kind == OUT_GEMV && bpad >= kTileBatch;
    for (int i = 0; mma && i < count; i++) mma = mma_eligible(ts[i]->d);
    // Activations in shared memory (one bulk copy per tensor per CTA) for a
    // single tensor, or when they are too large to stay in the L1 left beside
    // the staging buffers (over 16 KB); a grouped launch over tensors with
    // small activations reads them through L1 instead of copying them for
    // every tensor a CTA touches (Phi-3-shaped step -3 %, one 4096-column
    // tensor +7 % if read through L1).
    long long x_elems = (out_kind == OUT_GEMV && !mma && max_kb <= kXSmemElems &&
                         (count == 1 || max_kb * 2 > kXL1Bytes))
                            ? max_kb
                            : 0;
    const int stage_rows = max_words + kSlackRows;
    // the run ring: kRing runs of 8 codes per lane (padded for the tensor-core GEMV's cross-warp reads)
    const int out_words = mma ? tile_ring_words(bits, lanes) : kRing * lanes * bits / 4;
    long long chunks = 0;
    for (int i = 0; i < count; i++) chunks += ts[i]->d.n_chunks;
    // Spread the chunks evenly over the SMs: small inputs get one CTA per SM
    // with one warp per chunk; large ones run persistent CTAs of 16 warps.
    const int wave_warps = (int)std::min<long long>(kMaxWarps, std::max<long long>(1, (chunks + di.sms - 1) / di.sms));
    LanesFn fn = mma ? pick_mma(bits, slow, lanes, batch) : pick_lanes(bits, out_kind, slow, bpad, lanes);
    if (!fn) return ENTRO_E_INVAL;  // a batched GEMV whose chunks are not whole rows
    // When every warp gets one chunk in a single wave, the chunks go to two
    // CTAs of half the warps per SM rather than one (the lockstep tensor-core
    // GEMV excepted): an SM then frees half its slots as soon as one of the
    // two finishes, and with launch overlap the next launch's CTA starts there
    // sooner (4096x4096 4-bit tensor: codes 9.0 -> 8.4 us, bf16 11.0 -> 10.8
    // us).  Kept only if two such CTAs fit on an SM.
    const bool may_halve = !mma && wave_warps > 1 && wave_warps < kMaxWarps;
    SmemOffsets so;
    int warps = 0, per_sm = 0;
    for (int attempt = may_halve ? 0 : 1; attempt < 2; attempt++) {
        warps = attempt == 0 ? (wave_warps + 1) / 2 : wave_warps;
        for (;;) {
            so = smem_layout(warps, x_elems, stage_rows * lanes, out_words,
                             mma ? static_cast<size_t>(warps) * mma_batch_tiles(batch) * 32 * 16 : 0,
                             mma ? kLutSize * 4 : kWideLutBytes);
            if ((long long)so.total <= di.smem_optin) break;
            if (warps > 1) warps--;
            else if (x_elems) { x_elems = 0; warps = kMaxWarps; }
            else return ENTRO_E_LIMIT;
        }
        if (kernel_config(reinterpret_cast<const void *>(fn), ts[0]->device, warps * 32, so.total, &per_sm) != ENTRO_OK)
            return ENTRO_E_CUDA;
        if (attempt == 1 || per_sm >= 2) break;
    }
    const size_t bytes = so.total;
    long long grid = std::min<long long>((chunks + warps - 1) / warps, (long long)per_sm * di.sms);
    grid = std::max<long long>(grid, 1);
    // overlap only with one or two (large) CTAs per SM: a later launch's CTAs
    // then take only slots that this launch's CTAs have left
    const bool overlap_ok = per_sm <= 2;
    LaunchArgs a;
    std::memset(&a, 0, sizeof(a));
    a.table = d_table;
    a.one = one;
    a.count = count;
    a.batch = batch;
    a.x_in_smem = x_elems > 0;
    a.stage_rows = stage_rows;
    a.out_words = out_words;
    a.x_elems = x_elems;
    a.total_syms = total;
    a.status = status;
    a.tx_extra = g_tx_extra.load(std::memory_order_relaxed);
    a.k_one = 1;
    const cudaError_t e = launch(fn, (unsigned)grid, warps * 32, bytes, st, a, overlap_ok);
    return e == cudaSuccess ? ENTRO_OK : cuda_fail(e, "lanes kernel launch");
}

template <int BITS, int OUT, int LANES, bool CO>
static LanesFn pick_rows3(bool slow, int nb) {
    if constexpr (OUT == OUT_GEMV) {
        if (nb == 2)
            return slow ? rows_kernel<BITS, OUT, true, LANES, 2, CO> : rows_kernel<BITS, OUT, false, LANES, 2, CO>;
    }
    return slow ? rows_kernel<BITS, OUT, true, LANES, 1, CO> : rows_kernel<BITS, OUT, false, LANES, 1, CO>;
}

template <int BITS, int LANES, bool CO>
static LanesFn pick_rows2(int out, bool slow, int nb) {
    if (out == OUT_CODES) return pick_rows3<BITS, OUT_CODES, LANES, CO>(slow, nb);
    if (out == OUT_BF16) return pick_rows3<BITS, OUT_BF16, LANES, CO>(slow, nb);
    return pick_rows3<BITS, OUT_GEMV, LANES, CO>(slow, nb);
}

// consumption order: 32-lane tiles only (one lane per thread)
static LanesFn pick_rows(int bits, int out, bool slow, int nb, int lanes, bool co) {
    if (co) return bits == 4 ? pick_rows2<4, 32, true>(out, slow, nb) : pick_rows2<8, 32, true>(out, slow, nb);
    if (bits == 4)
        return lanes == 64 ? pick_rows2<4, 64, false>(out, slow, nb) : pick_rows2<4, 32, false>(out, slow, nb);
    return lanes == 64 ? pick_rows2<8, 64, false>(out, slow, nb) : pick_rows2<8, 32, false>(out, slow, nb);
}

// Launch the row-tile kernel over `count` entries (table on device, or `one`).
static int launch_rows(const TensorHandle *const *ts, int count, int out_kind, int batch, const GroupEntry *d_table,
                       const GroupEntry &one, int32_t *status, cudaStream_t st) {
    bool slow = false;
    const int bits = ts[0]->d.bits, lanes = ts[0]->d.lanes, format = ts[0]->d.format;
    const bool co = format == ENTRO_FORMAT_ROWS_CO;
    if (co && lanes != 32) return ENTRO_E_INVAL;
    int max_words = 0;
    long long max_runs = 0, total = 0, units = 0;
    for (int i = 0; i < count; i++) {
        const DevTensor &d = ts[i]->d;
        if (d.format != format || d.bits != bits || d.lanes != lanes) return ENTRO_E_INVAL;
        slow = slow || ts[i]->slow;
        max_words = std::max(max_words, d.max_chunk_words);
        max_runs = std::max(max_runs, d.chunk_symbols / lanes / kRun);
        total += d.n;
        units += d.n_chunks;  // tiles
    }
    if (total == 0) return ENTRO_OK;
    DeviceInfo di;
    if (device_info(ts[0]->device, &di) != ENTRO_OK) return ENTRO_E_CUDA;
    const int nb = out_kind == OUT_GEMV && batch > 8 ? 2 : 1;
    LanesFn fn = pick_rows(bits, out_kind, slow, nb, lanes, co);
    const int stage_rows = max_words + kSlackRows;
    // a run slot for every run of a chunk, plus the runs a lane may complete past its last check
    int run_buf_bytes = static_cast<int>(max_runs + wide_runs_per_check(bits, 8)) * rows_run_bytes(bits, lanes);
    // the GEMV parks two sets of partial sums (fp32 D fragments) in a warp's run buffer
    if (out_kind == OUT_GEMV) run_buf_bytes = std::max(run_buf_bytes, 2 * (lanes / 16) * nb * 4 * 32 * 4);
    int warps = (int)std::min<long long>(kMaxWarps, std::max<long long>(1, (units + di.sms - 1) / di.sms));
    RowsLayout rl;
    for (;;) {
        rl = rows_layout(warps, stage_rows * lanes, run_buf_bytes);
        if ((long long)rl.total <= di.smem_optin) break;
        if (warps > 1) warps--;
        else return ENTRO_E_LIMIT;
    }
    int per_sm = 0;
    if (kernel_config(reinterpret_cast<const void *>(fn), ts[0]->device, warps * 32, rl.total, &per_sm) != ENTRO_OK)
        return ENTRO_E_CUDA;
    long long grid = std::min<long long>((units + warps - 1) / warps, (long long)per_sm * di.sms);
    grid = std::max<long long>(grid, 1);
    LaunchArgs a;
    std::memset(&a, 0, sizeof(a));
    a.table = d_table;
    a.one = one;
    a.count = count;
    a.batch = batch;
    a.stage_rows = stage_rows;
    a.out_words = run_buf_bytes / 4;
    a.total_syms = total;
    a.status = status;
    a.tx_extra = g_tx_extra.load(std::memory_order_relaxed);
    a.k_one = 1;
    const cudaError_t e = launch(fn, (unsigned)grid, warps * 32, rl.total, st, a, per_sm <= 2);
    return e == cudaSuccess ? ENTRO_OK : cuda_fail(e, "row-tile kernel launch");
}

// A grouped launch of tensors of one format.
static int launch_group(const TensorHandle *const *ts, int count, int out_kind, int batch, const GroupEntry *d_table,
                        const GroupEntry &one, int32_t *status, cudaStream_t st) {
    if (ts[0]->d.format == ENTRO_FORMAT_ROWS || ts[0]->d.format == ENTRO_FORMAT_ROWS_CO)
        return launch_rows(ts, count, out_kind, batch, d_table, one, status, st);
    return launch_lanes(ts, count, out_kind, batch, d_table, one, status, st);
}

static LanesFn pick_segment(int bits, int out, bool slow) {
    if (bits == 4) {
        if (out == OUT_CODES) return slow ? segment_kernel<4, OUT_CODES, true> : segment_kernel<4, OUT_CODES, false>;
        return slow ? segment_kernel<4, OUT_BF16, true> : segment_kernel<4, OUT_BF16, false>;
    }
    if (out == OUT_CODES) return slow ? segment_kernel<8, OUT_CODES, true> : segment_kernel<8, OUT_CODES, false>;
    return slow ? segment_kernel<8, OUT_BF16, true> : segment_kernel<8, OUT_BF16, false>;
}

static int launch_single(const TensorHandle *t, int out_kind, void *out, int32_t *status, cudaStream_t st) {
    const DevTensor &d = t->d;
    if (d.n_chunks == 0) return ENTRO_OK;
    DeviceInfo di;
    if (device_info(t->device, &di) != ENTRO_OK) return ENTRO_E_CUDA;
    // chunks of up to kSegChunkSymbols codes: a CTA per chunk, staged in shared memory
    const int stage_words = ((d.max_chunk_words + 12) + 3) & ~3;
    const SegLayout sl = seg_layout(stage_words, static_cast<int>(d.chunk_symbols));
    if (d.chunk_symbols <= kSegChunkSymbols && (long long)sl.total <= di.smem_optin) {
        LanesFn fn = pick_segment(d.bits, out_kind, t->slow);
        int per_sm = 0;
        if (kernel_config(reinterpret_cast<const void *>(fn), t->device, kSegThreads, sl.total, &per_sm) != ENTRO_OK)
            return ENTRO_E_CUDA;
        LaunchArgs a;
        std::memset(&a, 0, sizeof(a));
        a.one.d = d;
        a.one.out = out;
        a.count = 1;
        a.batch = 1;
        a.stage_rows = stage_words;
        a.status = status;
        a.tx_extra = g_tx_extra.load(std::memory_order_relaxed);
        const cudaError_t e = launch(fn, (unsigned)d.n_chunks, kSegThreads, sl.total, st, a, false);
        return e == cudaSuccess ? ENTRO_OK : cuda_fail(e, "segment kernel launch");
    }
    LanesFn fn = pick_single(d.bits, out_kind, t->slow);
    const size_t bytes = smem_layout(0, 0, 0, 0).total;
    const int threads = 64;  // two chunks per CTA: spreads small tensors over the SMs
    int per_sm = 0;
    if (kernel_config(reinterpret_cast<const void *>(fn), t->device, threads, bytes, &per_sm) != ENTRO_OK)
        return ENTRO_E_CUDA;
    LaunchArgs a;
    std::memset(&a, 0, sizeof(a));
    a.one.d = d;
    a.one.out = out;
    a.count = 1;
    a.batch = 1;
    a.status = status;
    a.tx_extra = g_tx_extra.load(std::memory_order_relaxed);
    const long long grid = (d.n_chunks * 32 + threads - 1) / threads;
    const cudaError_t e = launch(fn, (unsigned)grid, threads, bytes, st, a, false);
    return e == cudaSuccess ? ENTRO_OK : cuda_fail(e, "single kernel launch");
}

static int decode_one(const entro_tensor *tensor, int out_kind, void *out, int32_t *status, void *stream) {
    if (!tensor) return ENTRO_E_INVAL;
    const TensorHandle *t = reinterpret_cast<const TensorHandle *>(tensor);
    if (t->d.n == 0) return ENTRO_OK;  // nothing to decode; `out` may be null
    if (!out) return ENTRO_E_INVAL;
    if (reinterpret_cast<uintptr_t>(out) & 15) return ENTRO_E_INVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (t->d.format == ENTRO_FORMAT_SINGLE) {
        if (out_kind == OUT_CODES && t->d.bits == 4 && (t->d.chunk_symbols & 1)) return ENTRO_E_INVAL;
        return launch_single(t, out_kind, out, status, st);
    }
    GroupEntry one;
    std::memset(&one, 0, sizeof(one));
    one.d = t->d;
    one.out = out;
    return launch_group(&t, 1, out_kind, 1, nullptr, one, status, st);
}

static int gemv_check(const TensorHandle *t, const void *x, int batch, const float *y) {
    if (!t || !x || !y || batch < 1 || batch > kMaxBatch) return ENTRO_E_INVAL;
    if (reinterpret_cast<uintptr_t>(x) & 15) return ENTRO_E_INVAL;
    const DevTensor &d = t->d;
    if (d.format == ENTRO_FORMAT_ROWS || d.format == ENTRO_FORMAT_ROWS_CO)
        return ENTRO_OK;  // any shape of the formats (cols a multiple of 8)
    if (d.format != ENTRO_FORMAT_LANES) return ENTRO_E_INVAL;
    if (d.cols <= 0 || d.cols % (kRun * d.lanes) || d.chunk_symbols % d.cols) return ENTRO_E_INVAL;
    return ENTRO_OK;
}

}  // namespace entro

extern "C" int entro_decode_codes(const entro_tensor *t, void *d_out, int32_t *d_status, void *stream) {
    return decode_one(t, OUT_CODES, d_out, d_status, stream);
}

extern "C" int entro_decode_dequant_bf16(const entro_tensor *t, void *d_out, int32_t *d_status, void *stream) {
    return decode_one(t, OUT_BF16, d_out, d_status, stream);
}

extern "C" int entro_decode_gemv(const entro_tensor *tensor, const void *d_x, int32_t batch, float *d_y,
                                 int32_t *d_status, void *stream) {
    const TensorHandle *t = reinterpret_cast<const TensorHandle *>(tensor);
    int r = gemv_check(t, d_x, batch, d_y);
    if (r != ENTRO_OK) return r;
    GroupEntry one;
    std::memset(&one, 0, sizeof(one));
    one.d = t->d;
    one.x = static_cast<const __nv_bfloat16 *>(d_x);
    one.y = d_y;
    return launch_group(&t, 1, OUT_GEMV, batch, nullptr, one, d_status, static_cast<cudaStream_t>(stream));
}

namespace entro {
struct GroupHandle {
    std::vector<const TensorHandle *> ts;
    GroupEntry first;
    const GroupEntry *d_table;
    int kind;
    int batch;
};
}  // namespace entro

extern "C" uint64_t entro_group_table_bytes(int32_t count) {
    return count > 0 ? align256(sizeof(GroupEntry) * (uint64_t)count) : 0;
}

extern "C" int entro_group_prepare(const entro_tensor *const *tensors, int32_t count, int32_t kind,
                                   const void *const *xs, float *const *ys, void *const *outs, int32_t batch,
                                   void *d_table, uint64_t table_bytes, void *stream, entro_group **out) {
    if (!out) return ENTRO_E_INVAL;
    *out = nullptr;
    if (!tensors || count < 1 || !d_table || (reinterpret_cast<uintptr_t>(d_table) & 255)) return ENTRO_E_INVAL;
    if (kind != ENTRO_GROUP_GEMV && kind != ENTRO_GROUP_BF16) return ENTRO_E_INVAL;
    if (table_bytes < entro_group_table_bytes(count)) return ENTRO_E_INVAL;
    const int out_kind = kind == ENTRO_GROUP_GEMV ? OUT_GEMV : OUT_BF16;
    if (out_kind == OUT_GEMV && (!xs || !ys)) return ENTRO_E_INVAL;
    if (out_kind == OUT_BF16 && !outs) return ENTRO_E_INVAL;
    GroupHandle *h = new (std::nothrow) GroupHandle();
    if (!h) return ENTRO_E_NOMEM;
    std::vector<GroupEntry> host((size_t)count);
    h->ts.resize((size_t)count);
    long long chunks = 0, syms = 0;
    for (int i = 0; i < count; i++) {
        const TensorHandle *t = reinterpret_cast<const TensorHandle *>(tensors[i]);
        int r = ENTRO_OK;
        if (!t || t->d.format == ENTRO_FORMAT_SINGLE) r = ENTRO_E_INVAL;
        else if (out_kind == OUT_GEMV) r = gemv_check(t, xs[i], batch, ys[i]);
        else if (!outs[i] || (reinterpret_cast<uintptr_t>(outs[i]) & 15)) r = ENTRO_E_INVAL;
        if (r == ENTRO_OK && i > 0 &&
            (t->device != h->ts[0]->device || t->d.bits != h->ts[0]->d.bits || t->d.format != h->ts[0]->d.format ||
             t->d.lanes != h->ts[0]->d.lanes))
            r = ENTRO_E_INVAL;
        if (r != ENTRO_OK) {
            delete h;
            return r;
        }
        h->ts[i] = t;
        GroupEntry &g = host[i];
        std::memset(&g, 0, sizeof(g));
        g.d = t->d;
        if (out_kind == OUT_GEMV) {
            g.x = static_cast<const __nv_bfloat16 *>(xs[i]);
            g.y = ys[i];
        } else {
            g.out = outs[i];
        }
        g.chunk_begin = chunks;
        g.sym_begin = syms;
        chunks += t->d.n_chunks;
        syms += t->d.n;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(d_table, host.data(), sizeof(GroupEntry) * (size_t)count, cudaMemcpyHostToDevice, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        delete h;
        return ENTRO_E_CUDA;
    }
    h->first = host[0];
    h->d_table = static_cast<const GroupEntry *>(d_table);
    h->kind = out_kind;
    h->batch = out_kind == OUT_GEMV ? batch : 1;
    *out = reinterpret_cast<entro_group *>(h);
    return ENTRO_OK;
}

extern "C" int entro_group_launch(const entro_group *group, int32_t *d_status, void *stream) {
    if (!group) return ENTRO_E_INVAL;
    const GroupHandle *h = reinterpret_cast<const GroupHandle *>(group);
    return launch_group(h->ts.data(), (int)h->ts.size(), h->kind, h->batch, h->d_table, h->first, d_status,
                        static_cast<cudaStream_t>(stream));
}

extern "C" void entro_group_free(entro_group *group) { delete reinterpret_cast<GroupHandle *>(group); }

// ------------------------------------------------------------------ grouped GEMV without allocation
//
// Some callers may not allocate device memory at all -- for instance code that
// runs inside a caching allocator's own hooks, or a serving runtime that
// reserves all device memory up front and forbids cudaMalloc afterwards.  For
// them the grouped GEMV can take its work table from a fixed array inside the
// library instead of from caller memory.  The array costs every GPU that loads
// the library kStaticGroupMax * sizeof(GroupEntry) bytes until process exit.

namespace entro {
constexpr int kStaticGroupMax = ENTRO_STATIC_GROUP_MAX;
constexpr int kStaticBatchCopy = 32;  // entries staged per host-to-device copy (a stack buffer)
static __device__ __align__(256) GroupEntry g_static_table[kStaticGroupMax];
// Device address of g_static_table, per device; the host-side name is only a
// stand-in, so the address comes from cudaGetSymbolAddress on first use.
static void *g_static_addr[kMaxDevices];
}  // namespace entro

extern "C" int entro_decode_gemv_group_static(const entro_tensor *const *tensors, const void *const *xs,
                                              float *const *ys, int32_t count, int32_t batch, int32_t *d_status,
                                              void *stream) {
    if (!tensors || !xs || !ys || count < 1) return ENTRO_E_INVAL;
    if (count > kStaticGroupMax) {
        snprintf(g_cuda_msg, sizeof(g_cuda_msg), "entro_decode_gemv_group_static: %d tensors exceed the fixed table "
                 "of %d entries", (int)count, kStaticGroupMax);
        return ENTRO_E_LIMIT;
    }
    const TensorHandle *const *ts = reinterpret_cast<const TensorHandle *const *>(tensors);
    for (int i = 0; i < count; i++) {
        const TensorHandle *t = ts[i];
        if (!t || t->d.format == ENTRO_FORMAT_SINGLE) return ENTRO_E_INVAL;
        const int r = gemv_check(t, xs[i], batch, ys[i]);
        if (r != ENTRO_OK) return r;
        if (t->device != ts[0]->device || t->d.bits != ts[0]->d.bits || t->d.format != ts[0]->d.format ||
            t->d.lanes != ts[0]->d.lanes)
            return ENTRO_E_INVAL;
    }
    const int dev = ts[0]->device;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess || cur != dev || dev >= kMaxDevices) return ENTRO_E_INVAL;
    void *table = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_static_addr[dev]) {
            void *p = nullptr;
            const cudaError_t e = cudaGetSymbolAddress(&p, g_static_table);
            if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
            g_static_addr[dev] = p;
        }
        table = g_static_addr[dev];
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    GroupEntry stage[kStaticBatchCopy];
    GroupEntry first;
    long long chunks = 0, syms = 0;
    for (int i0 = 0; i0 < count; i0 += kStaticBatchCopy) {
        const int m = std::min(kStaticBatchCopy, count - i0);
        for (int k = 0; k < m; k++) {
            const TensorHandle *t = ts[i0 + k];
            GroupEntry &g = stage[k];
            std::memset(&g, 0, sizeof(g));
            g.d = t->d;
            g.x = static_cast<const __nv_bfloat16 *>(xs[i0 + k]);
            g.y = ys[i0 + k];
            g.chunk_begin = chunks;
            g.sym_begin = syms;
            chunks += t->d.n_chunks;
            syms += t->d.n;
        }
        if (i0 == 0) first = stage[0];
        // pageable source: the call returns once `stage` has been consumed
        const cudaError_t e = cudaMemcpyAsync(static_cast<GroupEntry *>(table) + i0, stage, sizeof(GroupEntry) * m,
                                              cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync (static group table)");
    }
    return launch_group(ts, count, OUT_GEMV, batch, static_cast<const GroupEntry *>(table), first, d_status, st);
}

extern "C" const char *entro_strerror(int code) {
    switch (code) {
        case ENTRO_OK: return "ok";
        case ENTRO_E_INVAL: return "invalid argument";
        case ENTRO_E_LIMIT: return "outside a documented limit";
        case ENTRO_E_FORMAT: return "malformed blob";
        case ENTRO_E_CORRUPT: return "corrupt coded data (no code matches)";
        case ENTRO_E_OVERRUN: return "coded stream ran past its chunk";
        case ENTRO_E_NOMEM: return "out of host memory";
        case ENTRO_E_CUDA: return "CUDA runtime error";
        case ENTRO_E_TIMEOUT: return "bounded wait on a copy gave up";
        default: return "unknown error";
    }
}

extern "C" int entro_version(void) { return 100; }

extern "C" ENTRO_API int entro_set_overlap(int enable) { return entro::g_overlap.exchange(enable ? 1 : 0); }

extern "C" ENTRO_API uint32_t entro_test_stall_tables(uint32_t extra_bytes) {
    return entro::g_tx_extra.exchange(extra_bytes);
}

extern "C" const char *entro_last_cuda_error(void) { return g_cuda_msg; }
