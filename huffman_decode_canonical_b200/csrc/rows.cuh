// rows.cuh -- the row-tile format on sm_100a: one kernel for codes, bf16 and
// the fused GEMV, on the lane decoder of wide_decoder.cuh.
// Included by decode.cu inside namespace entro, after the shared helpers.
//
// Row tiles (a reading of the interleaved lanes of "LazyWeights:
// Decode-on-Demand Edge LLMs", arXiv 2611.17108v1, abstract, made for the
// matrix-vector product of token generation): a chunk is a tile of L = 32
// (or 64) rows by Kc = chunk_symbols / L columns, and lane l of the tile is
// row l.  One warp decodes a tile, so at run t every lane holds 8 codes of
// its own row at the same 8 columns:
//   * the GEMV needs no cross-lane reduction (a lane's row is its own), the
//     activations of run t are the same for the whole warp, and the decoded
//     weights of 16 rows x 8 columns are ready-made A fragments of the
//     tensor cores' m16n8k16 product (mma.sync, bf16 in, fp32 accumulate), so
//     one warp multiplies at any batch from 1 to 16 without waiting for other
//     warps;
//   * a warp takes consecutive tiles, so a row group's partial sums stay in
//     registers; a row group split between warps is summed in warp order (no
//     atomics; a fixed summation order).
//
// Decoding: the lane decoder of wide_decoder.cuh (two-word table entries, a
// counter register for window bits, pending bits and runs).  Every run of a
// chunk has its own slot in the warp's run buffer, at (run, lane) in output
// order, so a lane may decode ahead up to the chunk's end while the warp's
// slowest lane catches up.

constexpr int kRowsBlock = 8;  // runs per emission block

// The consumption-order format is defined by a reference decoder; this one must
// take the same codes per lookup and refill at the same points.
static_assert(kCoPeekBits == kMaxLutBits && kCoCodes4 == wide_max_codes(4) && kCoCodes8 == wide_max_codes(8),
              "consumption order: lookups as the format defines them");

// Run-buffer geometry: a run of every lane, then the next run.  4-bit: one
// word per lane, runs LANES + 8 words apart; 8-bit: two words per lane, runs
// 2 * (LANES + 4) words apart.  The pads put the slots that one fragment load
// of the tensor-core GEMV reads (lanes 8 apart, runs 1 apart) in different
// banks.
__host__ __device__ constexpr int rows_lane_bytes(int bits) { return bits == 4 ? 4 : 8; }
__host__ __device__ constexpr int rows_run_bytes(int bits, int lanes) {
    return bits == 4 ? 4 * (lanes + 8) : 8 * (lanes + 4);
}
// Slot of row l within a run.  quad (the 4-bit 32-row GEMV at batch 9-16):
// rows l, l + 8, l + 16, l + 24 are adjacent, so thread (gid, tig) fetches the
// four slots it feeds to the tensor cores (rows gid + 8 j at one run) with one
// 16-byte load, and a run's 32 slots stay in 32 different banks.  (At batch
// 1-8 the plain order measured faster.)
__host__ __device__ constexpr int rows_slot(bool quad, int l) { return quad ? 4 * (l & 7) + (l >> 3) : l; }

struct RowsLayout {
    size_t wlut, vtab, vpair, slow, tbar, tags, bars, stage, runs, total;
};

// Shared memory of the row-tile kernel: tables, barriers, per-warp double
// staging of chunk words and run buffer.
__host__ __device__ inline RowsLayout rows_layout(int warps, int stage_words, int run_buf_bytes) {
    RowsLayout o;
    size_t p = 0;
    o.wlut = p;
    p += kWideLutBytes;
    o.vtab = p;
    p += 256 * 4;
    o.vpair = p;
    p += 256 * 4;
    o.slow = p;
    p += kSlowBytes;
    o.tbar = p;
    p += 8;
    p = align_up(p, 16);
    o.tags = p;  // GEMV: per warp, the row groups of its first and last partial sums
    p += (size_t)kMaxWarps * 2 * 8;
    o.bars = p;
    p += (size_t)warps * 2 * 8;
    p = align_up(p, 128);
    o.stage = p;
    p += (size_t)warps * 2 * (size_t)stage_words * 4;
    p = align_up(p, 16);
    o.runs = p;
    p += (size_t)warps * (size_t)run_buf_bytes;
    o.total = align_up(p, 16);
    return o;
}

// the 8 4-bit codes of a run word -> 8 bf16 values (4 words, value of code i in half i)
__device__ __forceinline__ uint4 run_values4(uint32_t word, uint32_t vpair, const Pipes &k) {
    const uint32_t c = vpair_swizzle4(word);
    uint4 v;
    v.x = lds32(imad(byte_of(c, 0), k.four, vpair));
    v.y = lds32(imad(byte_of(c, 1), k.four, vpair));
    v.z = lds32(imad(byte_of(c, 2), k.four, vpair));
    v.w = lds32(imad(imulhi(c, k.two8), k.four, vpair));
    return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// 8 codes of a run slot -> 8 bf16 values (4 words, value of code i in half i)
template <int BITS>
__device__ __forceinline__ uint4 slot_values(uint32_t slot, uint32_t vtab, uint32_t vpair, const Pipes &k) {
    uint4 v;
    if (BITS == 4) {
        v = run_values4(lds32(slot), vpair, k);
    } else {
        const uint2 c = lds64(slot);
        auto val = [&](uint32_t b) { return lds32(imad(b, k.four, vtab)); };
        v.x = __byte_perm(val(byte_of(c.x, 0)), val(byte_of(c.x, 1)), 0x5410);
        v.y = __byte_perm(val(byte_of(c.x, 2)), val(imulhi(c.x, k.two8)), 0x5410);
        v.z = __byte_perm(val(byte_of(c.y, 0)), val(byte_of(c.y, 1)), 0x5410);
        v.w = __byte_perm(val(byte_of(c.y, 2)), val(imulhi(c.y, k.two8)), 0x5410);
    }
    return v;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Row-tile geometry of one tensor.
struct TileShape {
    long long K, Kc, T, G;  // columns, columns per tile, tiles per row group, row groups
};

__device__ __forceinline__ TileShape tile_shape(const DevTensor &d, int lanes) {
    TileShape s;
    s.K = d.cols;
    s.Kc = d.chunk_symbols / lanes;
    s.T = (s.K + s.Kc - 1) / s.Kc;
    s.G = (d.rows + lanes - 1) / lanes;
    return s;
}

// First tile whose first symbol is at or after symbol `off` of the tensor.
__device__ __forceinline__ long long tile_at(const DevTensor &d, const TileShape &s, int lanes, long long off) {
    if (off <= 0) return 0;
    if (off >= d.n) return d.n_chunks;
    const long long grp = off / (lanes * s.K);
    const long long rem = off - grp * lanes * s.K;
    const long long nr = min(static_cast<long long>(lanes), d.rows - grp * lanes);
    const long long j = (rem + nr * s.Kc - 1) / (nr * s.Kc);
    return j >= s.T ? (grp + 1) * s.T : grp * s.T + j;
}

// The table copies of one tensor, with `tx_extra` bytes that never arrive
// added to the barrier's count (a test of the bounded wait; 0 otherwise).
template <bool SLOW>
__device__ __forceinline__ void rows_issue_tables(const DevTensor &d, uint8_t *smem, const RowsLayout &L,
                                                  uint64_t *tbar, uint32_t tx_extra) {
    if (threadIdx.x != 0) return;
    uint32_t bytes = kWideLutBytes + tx_extra;
    if (SLOW) bytes += kSlowBytes;
    mbar_arrive_expect_tx(tbar, bytes);
    bulk_copy_g2s(smem + L.wlut, d.wlut, kWideLutBytes, tbar);
    if (SLOW) bulk_copy_g2s(smem + L.slow, d.slow_limit, kSlowBytes, tbar);
}

// y[b, row] from the D fragments of a row group: thread (gid, tig) holds rows
// gid and gid + 8 of each 16-row tile and batch columns 2 tig, 2 tig + 1.
template <int kMT, int NB>
__device__ __forceinline__ void rows_store_y(const GroupEntry &g, const DevTensor &d, int batch, long long row0,
                                             int gid, int tig, const float (&acc)[kMT][NB][4]) {
#pragma unroll
    for (int m = 0; m < kMT; m++)
#pragma unroll
        for (int nb = 0; nb < NB; nb++)
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const long long row = row0 + 16 * m + gid + 8 * (i >> 1);
                const int bb = 8 * nb + 2 * tig + (i & 1);
                if (row < d.rows && bb < batch) g.y[static_cast<long long>(bb) * d.rows + row] = acc[m][nb][i];
            }
}

// Row-tile kernel.  OUT_GEMV: the CTA's tiles of a tensor (row groups in order,
// column tiles within a group) are cut into one contiguous share per warp; a
// warp accumulates a row group's partial sums in registers over consecutive
// tiles and multiplies on the tensor cores (NB = 8-row tiles of the batch).  A
// row group whose tiles span several warps is finished after the tensor's
// barrier: the warp that began it adds the other warps' partial sums in warp
// order (a fixed order: results do not depend on timing).  OUT_CODES /
// OUT_BF16: warps take tiles in turn.
template <int BITS, int OUT, bool SLOW, int LANES, int NB, bool CO>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) rows_kernel(const __grid_constant__ LaunchArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    constexpr int LPT = LANES / kLanes;  // lanes (rows) per thread
    constexpr int kMT = LANES / 16;      // 16-row MMA tiles per row group
    constexpr int kStepsPerCheck = 8;
    constexpr int kUnit = CO ? 4 : LANES;  // chunk sizes are multiples of it
    constexpr bool kQuad = BITS == 4 && LANES == 32 && OUT == OUT_GEMV && NB == 2;  // slot order, see rows_slot
    constexpr bool kPreX = BITS == 4 && OUT == OUT_GEMV && NB == 1;  // activations loaded before a block's decode
    const int warps = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;  // MMA fragment coordinates
    const Pipes pk{a.k_one, a.k_one << 2, a.k_one << 3, a.k_one << 8, a.k_one << 12, a.k_one << 24};
    const RowsLayout L = rows_layout(warps, a.stage_rows * LANES, a.out_words * 4);
    uint64_t *tbar = reinterpret_cast<uint64_t *>(smem_raw + L.tbar);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem_raw + L.bars) + 2 * warp;
    const size_t buf_words = static_cast<size_t>(a.stage_rows) * LANES;
    uint32_t *stage = reinterpret_cast<uint32_t *>(smem_raw + L.stage) + static_cast<size_t>(warp) * 2 * buf_words;
    const uint32_t runbuf = smem_addr(smem_raw + L.runs) + static_cast<uint32_t>(warp * a.out_words * 4);
    const uint32_t wlut = smem_addr(smem_raw + L.wlut), vtab = smem_addr(smem_raw + L.vtab),
                   vpair = smem_addr(smem_raw + L.vpair);
    const uint32_t *slim = reinterpret_cast<const uint32_t *>(smem_raw + L.slow);
    const int32_t *soffs = reinterpret_cast<const int32_t *>(smem_raw + L.slow + 128);
    const uint8_t *ssyms = smem_raw + L.slow + 256;
    uint32_t *svtab = reinterpret_cast<uint32_t *>(smem_raw + L.vtab);
    uint32_t *svpair = reinterpret_cast<uint32_t *>(smem_raw + L.vpair);
    if (lane == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 1, 1);
    }
    if (threadIdx.x == 0) mbar_init(tbar, 1);
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
    uint32_t phase0 = 0, phase1 = 0, tphase = 0;
    bool dead = false;  // this warp gave up on a copy: it decodes nothing more but keeps the CTA's barriers
    for (; ei < a.count; ei++) {
        const GroupEntry &g = entry_at(a, ei);
        if (g.sym_begin >= s1) break;
        const DevTensor &d = g.d;
        const TileShape sh = tile_shape(d, LANES);
        // this CTA's tiles: GEMV, whole row groups whose first symbol lies in [s0, s1);
        // otherwise tiles whose first symbol does
        long long ua, ub;
        if (OUT == OUT_GEMV) {
            const long long gs = LANES * sh.K;  // symbols of a full row group
            ua = (s0 > g.sym_begin ? (s0 - g.sym_begin + gs - 1) / gs : 0) * sh.T;
            ub = min(sh.G, (s1 - g.sym_begin + gs - 1) / gs) * sh.T;
        } else {
            ua = tile_at(d, sh, LANES, s0 - g.sym_begin);
            ub = tile_at(d, sh, LANES, s1 - g.sym_begin);
        }
        if (ua >= ub) continue;
        // GEMV: warp w takes the contiguous tiles [wa, wb); otherwise tiles ua + w, ua + w + warps, ...
        const long long wa = ua + (ub - ua) * warp / warps, wb = ua + (ub - ua) * (warp + 1) / warps;
        auto chunk_of = [&](long long k) -> long long {
            if (OUT == OUT_GEMV) return wa + k < wb ? wa + k : -1;
            const long long c = ua + warp + k * warps;
            return c < ub ? c : -1;
        };
        rows_issue_tables<SLOW>(d, smem_raw, L, tbar, a.tx_extra);
        bool pend0 = false, pend1 = false;
        if (!dead) {
            const long long c0 = chunk_of(0), c1 = chunk_of(1);
            const long long cq = (lane < 2) ? c0 : c1;
            uint64_t iv = 0;
            if (lane < 4 && cq >= 0) iv = d.index[2 * cq + 2 * (lane & 1)];
            const uint64_t st0 = __shfl_sync(0xffffffffu, iv, 0), nx0 = __shfl_sync(0xffffffffu, iv, 1);
            const uint64_t st1 = __shfl_sync(0xffffffffu, iv, 2), nx1 = __shfl_sync(0xffffffffu, iv, 3);
            if (lane == 0) {
                if (c0 >= 0) issue_words(d, st0, nx0, stage, bar, a.stage_rows, LANES, kUnit);
                if (c1 >= 0) issue_words(d, st1, nx1, stage + buf_words, bar + 1, a.stage_rows, LANES, kUnit);
            }
            pend0 = c0 >= 0;
            pend1 = c1 >= 0;
        }
        grid_wait_prior();
        // dequantized values (EntroLLM: weights stay quantized codes until used)
        if (OUT != OUT_CODES) {
            for (int q = threadIdx.x; q < 256; q += blockDim.x) {
                svtab[q] = q < (1 << d.bits) ? dequant_bf16_bits(q, d.zero, d.scale) : 0u;
                if (BITS == 4)
                    svpair[vpair_index(q)] = dequant_bf16_bits(q & 15, d.zero, d.scale) |
                                (dequant_bf16_bits(q >> 4, d.zero, d.scale) << 16);
            }
        }
        const bool tables_ok = __syncthreads_and(mbar_wait(tbar, tphase & 1));
        tphase++;
        if (!tables_ok) {
            // the table barrier may never complete: give up on every later entry, let this
            // entry's copies land (bounded waits) and leave
            set_status(a.status, ENTRO_E_TIMEOUT);
            if (pend0) mbar_wait(bar, phase0 & 1);
            if (pend1) mbar_wait(bar + 1, phase1 & 1);
            if (threadIdx.x == 0) mbar_wait(tbar, (tphase - 1) & 1);
            __syncthreads();
            return;
        }
        const bool refill_each = SLOW && d.max_len > kCoRefillEachAbove;
        float acc[kMT][NB][4];
        float hacc[kMT][NB][4];           // partial sums of a row group begun by an earlier warp
        long long head_g = -1, tail_g = -1;  // row groups of this warp's partial sums (hacc, acc)
        bool began = false;               // the current row group began in this warp
        long long k = 0;
        // GEMV: the warp's tiles are consecutive, so their (row group, column tile) advance by one
        long long ggrp = OUT == OUT_GEMV ? wa / sh.T : 0, gj = OUT == OUT_GEMV ? wa % sh.T : 0;
        for (long long c = chunk_of(0); c >= 0 && !dead; c = chunk_of(++k)) {
            const int b = static_cast<int>(k & 1);
            const uint32_t phase = b ? phase1 : phase0;
            if (!__all_sync(0xffffffffu, mbar_wait(bar + b, phase & 1))) {
                set_status(a.status, ENTRO_E_TIMEOUT);
                dead = true;
                break;
            }
            if (b) { phase1++; pend1 = false; }
            else { phase0++; pend0 = false; }
            long long grp, j;
            if (OUT == OUT_GEMV) {
                grp = ggrp;
                j = gj;
                if (++gj == sh.T) {
                    gj = 0;
                    ggrp++;
                }
            } else {
                grp = c / sh.T;
                j = c - grp * sh.T;
            }
            const long long row0 = grp * LANES, col0 = j * sh.Kc;
            const int nrows = static_cast<int>(min(static_cast<long long>(LANES), d.rows - row0));
            const int runs = static_cast<int>(min(sh.Kc, sh.K - col0) / kRun);
            if (OUT == OUT_GEMV && (j == 0 || c == wa)) {
                began = j == 0;
#pragma unroll
                for (int m = 0; m < kMT; m++)
#pragma unroll
                    for (int nb = 0; nb < NB; nb++)
#pragma unroll
                        for (int i = 0; i < 4; i++) acc[m][nb][i] = 0.f;
            }
            const uint64_t wst = d.index[2 * c], wnx = d.index[2 * c + 2];
            // consumption order: a count header, then three rows of every lane's first words
            const int cbytes = CO ? co_count_bytes(static_cast<uint64_t>(sh.Kc), static_cast<uint32_t>(d.max_len)) : 0;
            const uint32_t hwords = CO ? static_cast<uint32_t>(co_header_words(LANES, cbytes)) : 0u;
            if (wnx >= wst && wnx <= static_cast<uint64_t>(d.payload_words) && (wnx - wst) % kUnit == 0 &&
                (!CO || wnx - wst >= hwords + 3u * LANES) &&
                (wnx - wst + LANES - 1) / LANES + kSlackRows <= static_cast<uint64_t>(a.stage_rows)) {
                const uint32_t *buf = stage + b * buf_words;
                const int words = static_cast<int>((wnx - wst) / LANES);
                WideDecoder<BITS, SLOW, LANES, rows_run_bytes(BITS, LANES), 0, CO> ld[LPT];
                uint32_t read_limit[LPT];
#pragma unroll
                for (int q = 0; q < LPT; q++) {
                    const int l = lane + kLanes * q;
                    if (CO) {
                        const uint32_t base = smem_addr(buf), cw = static_cast<uint32_t>(wnx - wst);
                        const uint8_t *hdr = reinterpret_cast<const uint8_t *>(buf);
                        const uint32_t nw = cbytes == 1 ? hdr[l] : hdr[2 * l] | (static_cast<uint32_t>(hdr[2 * l + 1]) << 8);
                        ld[q].init_co(pk, wlut, base + 4u * (hwords + l), runbuf + rows_slot(kQuad, l) * rows_lane_bytes(BITS),
                                      base + 4u * (hwords + 3u * LANES), nw > 3u ? nw - 3u : 0u, base + 4u * (cw - 1u),
                                      l < nrows);
                        read_limit[q] = base + 4u * cw;  // the cursor may end here, not past it
                    } else {
                        ld[q].init(pk, wlut, smem_addr(buf + l), runbuf + rows_slot(kQuad, l) * rows_lane_bytes(BITS),
                                   a.stage_rows - 1, l < nrows);
                        read_limit[q] = smem_addr(buf + l) + 4u * LANES * static_cast<uint32_t>(words + kOverrunRows);
                    }
                }
                // GEMV: this thread's row of x (batch row 8 nb + gid) at the tile's first column
                const __nv_bfloat16 *xrow[NB];
#pragma unroll
                for (int nb = 0; nb < NB; nb++)
                    xrow[nb] = OUT == OUT_GEMV ? g.x + min(8 * nb + gid, a.batch - 1) * sh.K + col0 : nullptr;
                const bool xlive0 = gid < a.batch;
                for (int tb = 0; tb < runs; tb += kRowsBlock) {
                    const int te = min(tb + kRowsBlock, runs);
                    // 4-bit GEMV at batch 1-8: the block's activations load while the block decodes
                    // (8-bit: measured no better)
                    uint4 xpre[kRowsBlock / 4];
                    if constexpr (kPreX) {
#pragma unroll
                        for (int gq = 0; gq < kRowsBlock / 4; gq++) {
                            const int tq = tb + 4 * gq + tig;
                            xpre[gq] = (tq < te && xlive0) ? ldg_nc_v4(xrow[0] + kRun * tq) : make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                    wide_decode_to<kStepsPerCheck>(ld, pk, slim, soffs, ssyms, te, runs, d.max_len, refill_each,
                                                   a.status);
                    __syncwarp();
                    constexpr uint32_t RB = rows_run_bytes(BITS, LANES), LB = rows_lane_bytes(BITS);
                    if (OUT == OUT_GEMV) {
                        // groups of 4 runs = 32 columns: thread (gid, tig) supplies run t0 + tig of
                        // rows gid and gid + 8 of each 16-row tile (A) and of batch row 8 nb + gid (B)
                        auto emit = [&](int t0, const uint4 (&xv)[NB]) {
                            const int t = t0 + tig;
                            if (kQuad) {
                                // the slots of rows gid, gid + 8, gid + 16, gid + 24 at run t
                                const uint4 w4 = lds128(runbuf + static_cast<uint32_t>(t) * RB + 16u * gid);
                                const uint32_t wr[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                                for (int m = 0; m < kMT; m++) {
                                    const uint4 wlo = run_values4(wr[2 * m], vpair, pk);
                                    const uint4 whi = run_values4(wr[2 * m + 1], vpair, pk);
#pragma unroll
                                    for (int nb = 0; nb < NB; nb++) {
                                        mma_16816_bf16(acc[m][nb], wlo.x, whi.x, wlo.y, whi.y, xv[nb].x, xv[nb].y);
                                        mma_16816_bf16(acc[m][nb], wlo.z, whi.z, wlo.w, whi.w, xv[nb].z, xv[nb].w);
                                    }
                                }
                            } else {
                                const uint32_t sl = runbuf + static_cast<uint32_t>(t) * RB + gid * LB;
#pragma unroll
                                for (int m = 0; m < kMT; m++) {
                                    const uint4 wlo = slot_values<BITS>(sl + 16 * m * LB, vtab, vpair, pk);
                                    const uint4 whi = slot_values<BITS>(sl + (16 * m + 8) * LB, vtab, vpair, pk);
#pragma unroll
                                    for (int nb = 0; nb < NB; nb++) {
                                        mma_16816_bf16(acc[m][nb], wlo.x, whi.x, wlo.y, whi.y, xv[nb].x, xv[nb].y);
                                        mma_16816_bf16(acc[m][nb], wlo.z, whi.z, wlo.w, whi.w, xv[nb].z, xv[nb].w);
                                    }
                                }
                            }
                        };
                        if constexpr (kPreX) {
#pragma unroll
                            for (int gq = 0; gq < kRowsBlock / 4; gq++) {
                                if (tb + 4 * gq >= te) break;
                                const uint4 xv[NB] = {xpre[gq]};
                                emit(tb + 4 * gq, xv);
                            }
                        } else {
                            for (int t0 = tb; t0 < te; t0 += 4) {
                                const int t = t0 + tig;
                                uint4 xv[NB];
#pragma unroll
                                for (int nb = 0; nb < NB; nb++)
                                    xv[nb] = (t < te && 8 * nb + gid < a.batch) ? ldg_nc_v4(xrow[nb] + kRun * t)
                                                                                : make_uint4(0u, 0u, 0u, 0u);
                                emit(t0, xv);
                            }
                        }
                    } else {
                        // thread (ll, tt) = (lane / 8, lane % 8) writes run tb + tt of rows ll, ll + 4, ...:
                        // 4 rows of 8 consecutive runs per warp store
                        const int ll = lane >> 3, t = tb + (lane & 7);
                        if (t < te) {
#pragma unroll 4
                            for (int l = ll; l < nrows; l += 4) {
                                const uint32_t sl = runbuf + static_cast<uint32_t>(t) * RB + l * LB;
                                const long long pos = (row0 + l) * sh.K + col0 + kRun * t;  // first code's index
                                if (OUT == OUT_BF16) {
                                    const uint4 v = slot_values<BITS>(sl, vtab, vpair, pk);
                                    *reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(g.out) + pos) = v;
                                } else if (BITS == 4) {
                                    reinterpret_cast<uint32_t *>(g.out)[pos >> 3] = lds32(sl);
                                } else {
                                    reinterpret_cast<uint2 *>(g.out)[pos >> 3] = lds64(sl);
                                }
                            }
                        }
                    }
                }
                bool ok = true;
#pragma unroll
                for (int q = 0; q < LPT; q++) {
                    if (CO) {
                        // every lane took all its words, and no more words than the chunk holds
                        if (ld[q].left != 0) set_status(a.status, ENTRO_E_CORRUPT);
                        ok = ok && ld[q].cur <= read_limit[q];
                    } else if (lane + kLanes * q < nrows) {
                        ok = ok && ld[q].bufa <= read_limit[q];
                    }
                }
                if (!ok) set_status(a.status, ENTRO_E_OVERRUN);
            } else {
                set_status(a.status, ENTRO_E_CORRUPT);
            }
            __syncwarp();  // run buffer and staging buffer are reused by the next chunks
            if (OUT == OUT_GEMV && (j == sh.T - 1 || c == wb - 1)) {
                if (began && j == sh.T - 1) {
                    rows_store_y(g, d, a.batch, row0, gid, tig, acc);
                } else if (!began) {
                    // begun by an earlier warp (only this warp's first row group can be)
                    head_g = grp;
#pragma unroll
                    for (int m = 0; m < kMT; m++)
#pragma unroll
                        for (int nb = 0; nb < NB; nb++)
#pragma unroll
                            for (int i = 0; i < 4; i++) hacc[m][nb][i] = acc[m][nb][i];
                } else {
                    tail_g = grp;  // continued by later warps (only this warp's last row group can be)
                }
            }
            const long long cn = chunk_of(k + 2);
            if (cn >= 0) {
                if (lane == 0) {
                    fence_proxy_async();
                    issue_chunk(d, cn, stage + b * buf_words, bar + b, a.stage_rows, LANES, kUnit);
                }
                if (b) pend1 = true;
                else pend0 = true;
            }
        }
        if (dead) {
            if (pend0) mbar_wait(bar, phase0 & 1);
            if (pend1) mbar_wait(bar + 1, phase1 & 1);
        }
        if (OUT == OUT_GEMV) {
            // partial sums into this warp's (now idle) run buffer: hacc, then acc, lane-major
            constexpr int kF = kMT * NB * 4;
            float *part = reinterpret_cast<float *>(smem_raw + L.runs + static_cast<size_t>(warp) * a.out_words * 4);
            long long *tags = reinterpret_cast<long long *>(smem_raw + L.tags);
#pragma unroll
            for (int m = 0; m < kMT; m++)
#pragma unroll
                for (int nb = 0; nb < NB; nb++)
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const int f = (m * NB + nb) * 4 + i;
                        if (head_g >= 0) part[f * 32 + lane] = hacc[m][nb][i];
                        if (tail_g >= 0) part[(kF + f) * 32 + lane] = acc[m][nb][i];
                    }
            if (lane == 0) {
                tags[2 * warp] = head_g;
                tags[2 * warp + 1] = tail_g;
            }
            __syncthreads();
            if (tail_g >= 0) {
                // this warp began row group tail_g: add the later warps' partial sums in warp order
                for (int w2 = warp + 1; w2 < warps && tags[2 * w2] == tail_g; w2++) {
                    const float *p2 =
                        reinterpret_cast<const float *>(smem_raw + L.runs + static_cast<size_t>(w2) * a.out_words * 4);
#pragma unroll
                    for (int m = 0; m < kMT; m++)
#pragma unroll
                        for (int nb = 0; nb < NB; nb++)
#pragma unroll
                            for (int i = 0; i < 4; i++) acc[m][nb][i] += p2[((m * NB + nb) * 4 + i) * 32 + lane];
                }
                rows_store_y(g, d, a.batch, tail_g * LANES, gid, tig, acc);
            }
        }
        __syncthreads();  // every warp done with this entry's tables and partial sums
    }
}
