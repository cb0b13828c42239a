// Prefill path: per-expert grouped GEMMs on the 5th-generation tensor cores.
//
// Rows of the grouped activation matrix follow the expert-sorted pair order
// (perm).  A tile is (expert e, up to 192 consecutive pair rows of e, 128
// output features).  The MMA runs "weights x activations": the 128 weight rows
// are the M side, the tile's pair rows the N side (N = rows rounded up to 16),
// so a lightly loaded expert wastes at most 15 columns.
//
//   GEMM1: D_g = W_g[rows] X^T, D_u = W_u[rows] X^T   (K = H)
//          h[pair][row] = bf16(silu(D_g) * D_u)
//   GEMM2: D = W_d[rows] h^T                           (K = I)
//          Y[pair][row] = bf16(w_pair * D)
//
// The dequantised weights never touch shared memory: they are written to
// tensor memory (tcgen05.st) and the MMA takes its A operand from there, so
// shared memory holds only the activation tiles and the tensor core reads
// only B from it.  TMEM (512 columns): the accumulators (gate and up for
// GEMM1, two buffers for GEMM2, PF_BN_MAX columns each) and, above them, a
// ring of A slots, each one stage (K = 64, 32 columns) of every weight matrix.
//
// A CTA owns one N-tile and a group of its M-tiles (GEMM1: one, GEMM2: eight);
// the CTAs of an N-tile are adjacent in launch order, so they run together and
// share its activation rows through L2.  Roles (736 threads):
//   warp 0      TMA loads of the activation tile (128-B swizzled K-major; a
//               tile of npad rows goes as at most one box each of 128, 64, 32
//               and 16 rows, since the TMA engine's cost grows with the
//               number of boxes);
//   warp 1      owns TMEM; one thread issues tcgen05.mma (GEMM1: for the gate
//               matrix, while a thread of warp 22 issues the up matrix's: one
//               thread issues at most one MMA per ~100 cycles, about 80 cycles
//               of tensor work at N = 160);
//   warps 2-5   drain finished accumulators (TMEM -> registers -> global; the
//               down GEMM double-buffers them so this overlaps the next
//               M-tile);
//   warps 6-21  load their own codes and scales from the arena, PF_PREFETCH
//               stages ahead in registers, and dequantise them into the A
//               slots (one 32-element block of 32 rows per warp and stage).
// Rings: full / empty (activation tiles), dequantised / free (A slots) and
// final / drained (accumulators) mbarriers; every wait is bounded.
#pragma once
#include "common.cuh"

#define PF_BK 64          // K elements per stage (one 128-byte swizzle row of bf16)
#define PF_BM 128         // weight rows per M-tile
#define PF_BN_MAX 192     // pair rows per tile (PREFILL_TILE_N)
#define PF_EPI_WARP0 2    // epilogue warps 2..5 (TMEM lane quadrants 2, 3, 0, 1)
#define PF_DQ_WARP0 6     // dequantisation warps 6..21 (four per TMEM lane quadrant)
#define PF_DQ_THREADS 512
#define PF_MMA2_WARP 22   // second MMA-issuing warp (GEMM1 up matrix)
#define PF_THREADS 736
#define PF_PREFETCH 4     // stages of codes and scales a dequantising thread holds ahead

template <int MODE>  // 0 = gate/up + SwiGLU, 1 = down + gate weight
struct PfCfg {
    static constexpr int NMAT = MODE == 0 ? 2 : 1;
    static constexpr int TSTAGES = 6;                            // ring of activation tiles
    static constexpr int NACC = MODE == 0 ? 1 : 2;               // accumulator buffers in TMEM
    static constexpr int MAT_COLS = PF_BN_MAX;                   // TMEM columns of one matrix's accumulator
    static constexpr int ACC_COLS = NMAT * PF_BN_MAX;            // TMEM columns of one accumulator buffer
    static constexpr int A_COL0 = NACC * ACC_COLS;               // first TMEM column of the A slots
    static constexpr int SLOT_COLS = NMAT * (PF_BK / 2);         // TMEM columns of one A slot (one stage)
    static constexpr int TMEM_COLS = 512;
    static constexpr int ASLOTS = (TMEM_COLS - A_COL0) / SLOT_COLS;  // 2 (GEMM1) or 4 (GEMM2)
    static constexpr int NISSUE = NMAT;                          // MMA-issuing threads, one per matrix
    // arrivals on a matrix's A slot: one dequant warp per (TMEM lane quadrant, half of the stage)
    static constexpr int DQ_ARRIVALS = 8;
    // The 4 epilogue warps drain the accumulators.  The last M-tile's drain is
    // the CTA's tail: the 16 dequant warps, done by then, take part (5 warps
    // per TMEM lane quadrant; only the epilogue warps arrive on "drained",
    // which nothing waits for after the last M-tile).  (Joining drains in the
    // middle of the dequant loop made GEMM1 slower: the drain's registers
    // spilled there.)
    static constexpr int TAIL_DRAIN_PARTS = 1 + PF_DQ_THREADS / 128;
    static constexpr int B_BYTES = PF_BN_MAX * PF_BK * 2;        // activation tile
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM = TSTAGES * B_BYTES + 1024 /*align*/ + PF_BN_MAX * 4 /*gate weights*/ + BAR_BYTES;
    static_assert(A_COL0 + ASLOTS * SLOT_COLS <= TMEM_COLS && ASLOTS >= 2, "TMEM budget");
    static_assert((2 * TSTAGES + 2 * NMAT * ASLOTS + 2 * NACC) * 8 + 4 <= BAR_BYTES, "barrier area");
    static_assert(PF_BK == 64 && TSTAGES * B_BYTES + 2048 < (1 << 18), "B descriptors as offsets of one base");
};

struct PrefillArgs {
    const uint8_t* arena;
    const int32_t* slot_table;
    int64_t n_slots;
    int64_t off_codes[3];
    int64_t off_scales[3];
    int64_t slot_bytes;
    int H, I, E, k, layer;
    int mgroups;             // CTAs per N-tile: each takes NOUT / PF_BM / mgroups consecutive M-tiles
    const int4* tiles;       // (expert, first pair row, rows, 0)
    const int32_t* meta;     // [1] = number of tiles
    const int32_t* perm;
    const float* topk_w;
    uint16_t* out;           // GEMM1: h [P][I]; GEMM2: Y [P][H]
};

// 8 codes (one 32-bit word of 4-bit codes, or 16 bits of 2-bit codes) ->
// 8 bf16 weights s * (q - offset), each rounded once from the exact product.
// q - offset is formed exactly in bf16 (128 + q by an exponent-bias bit
// pattern, then a subtraction).  The fp16 scale splits exactly into bf16
// s_hi + s_lo (11 significant bits = 8 + 3), (q - offset) * s_lo is exact,
// and one fused multiply-add adds (q - offset) * s_hi with a single rounding.
template <int BITS>
__device__ __forceinline__ uint4 dq8(uint32_t w, uint32_t s2hi, uint32_t s2lo) {
    constexpr uint32_t kMagic = 0x43004300u;                       // bf16 pair (128, 128)
    constexpr uint32_t kOff = BITS == 4 ? 0x43084308u : 0x43024302u;  // bf16 pair (136, 136) or (130, 130)
    uint32_t pr[4];
    // byte_perm selector: result byte 0 <- byte i of the first word, byte 2 <- byte i of the second
    if (BITS == 4) {
        // pair i = (low nibble, high nibble) of byte i
        const uint32_t w4 = w >> 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) pr[i] = (__byte_perm(w, w4, (uint32_t)(i | ((4 + i) << 8))) & 0x000F000Fu) | kMagic;
    } else {
        // byte i holds 4 codes at bit pairs 0-1, 2-3, 4-5, 6-7
        const uint32_t w2 = w >> 2, w4 = w >> 4, w6 = w >> 6;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            pr[2 * i] = (__byte_perm(w, w2, (uint32_t)(i | ((4 + i) << 8))) & 0x00030003u) | kMagic;
            pr[2 * i + 1] = (__byte_perm(w4, w6, (uint32_t)(i | ((4 + i) << 8))) & 0x00030003u) | kMagic;
        }
    }
    uint4 r;
    uint32_t* rr = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&pr[i]);
        __nv_bfloat162 o = *reinterpret_cast<const __nv_bfloat162*>(&kOff);
        __nv_bfloat162 shi = *reinterpret_cast<__nv_bfloat162*>(&s2hi);
        __nv_bfloat162 slo = *reinterpret_cast<__nv_bfloat162*>(&s2lo);
        __nv_bfloat162 q = __hsub2(v, o);                    // exact: small integers
        __nv_bfloat162 d = __hfma2(q, shi, __hmul2(q, slo));  // exact low part, one rounding
        rr[i] = *reinterpret_cast<uint32_t*>(&d);
    }
    return r;
}

// Codes of one 32-element block of one row: 16 bytes (4-bit) or 8 (2-bit, in .x and .y).
template <int BITS>
__device__ __forceinline__ uint4 load_block_codes(const uint8_t* p) {
    if (BITS == 4) return __ldg(reinterpret_cast<const uint4*>(p));
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    return make_uint4(v.x, v.y, 0u, 0u);
}

// One 32-element block of one row, codes in registers -> 16 columns of bf16
// pairs (elements 2c, 2c + 1 in column c), the TMEM layout of an A row.
template <int BITS>
__device__ __forceinline__ void dequant_block_cols(uint4 c, float s, uint32_t (&col)[16]) {
    uint32_t w[4];
    if (BITS == 4) {
        w[0] = c.x; w[1] = c.y; w[2] = c.z; w[3] = c.w;
    } else {
        w[0] = c.x & 0xffffu; w[1] = c.x >> 16; w[2] = c.y & 0xffffu; w[3] = c.y >> 16;
    }
    const float shi = __bfloat162float(__float2bfloat16_rn(s));
    const uint32_t s2hi = pack_bf16x2(shi, shi), s2lo = pack_bf16x2(s - shi, s - shi);  // both exact
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {  // elements 8cc..8cc+7 -> columns 4cc..4cc+3
        const uint4 v = dq8<BITS>(w[cc], s2hi, s2lo);
        col[4 * cc + 0] = v.x; col[4 * cc + 1] = v.y; col[4 * cc + 2] = v.z; col[4 * cc + 3] = v.w;
    }
}

// One CTA per (N-tile, M-tile group): expert e, rows row0 .. row0+nrows of the
// grouped activations, M-tiles mt0 .. mt0+nmt of the output features.  Stage i
// covers (M-tile mt0 + i / nk, K-block i % nk) and A slot i % ASLOTS.  The four tensor maps view the same activation matrix with boxes of
// 128, 64, 32 and 16 rows.
template <int MODE, int B0, int B1>
__global__ void __launch_bounds__(PF_THREADS, 1)
    k_prefill_gemm(const __grid_constant__ CUtensorMap tx128, const __grid_constant__ CUtensorMap tx64,
                   const __grid_constant__ CUtensorMap tx32, const __grid_constant__ CUtensorMap tx16, PrefillArgs a) {
    using C = PfCfg<MODE>;
    // CTA b serves N-tile b / mgroups and its M-tile group b % mgroups: the CTAs
    // sharing an activation tile are adjacent in launch order, so they run
    // together and its re-reads are served by L2.
    const int tile = blockIdx.x / a.mgroups, mgrp = blockIdx.x % a.mgroups;
    if (tile >= a.meta[1]) return;
    const int4 td = a.tiles[tile];
    const int e = td.x, row0 = td.y, nrows = td.z;
    const int npad = (nrows + 15) & ~15;
    const int K = MODE == 0 ? a.H : a.I;
    const int NOUT = MODE == 0 ? a.I : a.H;  // output features (row length of `out`)
    const int nk = K / PF_BK, nmt = NOUT / PF_BM / a.mgroups, mt0 = mgrp * nmt, nstage = nk * nmt;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* sB = smem;                                            // [TSTAGES][B_BYTES]
    float* s_w = reinterpret_cast<float*>(sB + C::TSTAGES * C::B_BYTES);  // [PF_BN_MAX] gate weights
    uint64_t* bars = reinterpret_cast<uint64_t*>(s_w + PF_BN_MAX);
    uint64_t* full = bars;                      // [TSTAGES] activation tile landed
    uint64_t* empty = full + C::TSTAGES;        // [TSTAGES] MMA done reading the activation tile
    uint64_t* deq = empty + C::TSTAGES;         // [NMAT][ASLOTS] A slot of a matrix written
    uint64_t* aempty = deq + C::NMAT * C::ASLOTS;  // [NMAT][ASLOTS] MMA done reading it
    uint64_t* accf = aempty + C::NMAT * C::ASLOTS;  // [NACC] accumulator final
    uint64_t* acce = accf + C::NACC;            // [NACC] accumulator drained
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + C::NACC);

    const int64_t slot = a.slot_table[(int64_t)a.layer * a.E + e];
    if (slot < 0 || slot >= a.n_slots) {  // expert without weights here contributes zero
        if (threadIdx.x == 0 && slot != MOE_SLOT_REMOTE) moe_set_status(MOE_ERR_SLOT);
        for (int i = threadIdx.x; i < nrows * NOUT; i += blockDim.x)
            a.out[(size_t)(row0 + i / NOUT) * NOUT + i % NOUT] = 0;
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::TSTAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::NISSUE);
        }
        for (int s = 0; s < C::NMAT * C::ASLOTS; ++s) {
            mbar_init(&deq[s], C::DQ_ARRIVALS);
            mbar_init(&aempty[s], 1);
        }
        for (int b = 0; b < C::NACC; ++b) {
            mbar_init(&accf[b], C::NISSUE);
            mbar_init(&acce[b], 4);
        }
        fence_mbar_init();
    }
    if (MODE == 1)
        for (int n = threadIdx.x; n < nrows; n += blockDim.x) s_w[n] = __ldg(a.topk_w + a.perm[row0 + n]);
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool alive = true;

    // Drains M-tile mt's accumulator from this warp's TMEM lane quadrant:
    // chunks part, part + nparts, ... of 16 columns (the next chunk loads while
    // one is stored), then one arrival on the accumulator's "drained" barrier.
    // Lane l holds output feature 32 q + l of the M-tile; neighbouring lanes
    // swap values so that each stores a bf16 pair: the even lane features
    // (l, l + 1) of row j, the odd lane features (l - 1, l) of row j + 1.
    auto drain = [&](int mt, int part, int nparts, bool arrive) -> bool {
        const int q = warp & 3, odd = lane & 1;
        const int buf = mt % C::NACC, use = mt / C::NACC;
        if (!mbar_wait_fast(&accf[buf], use & 1)) return false;
        __syncwarp();  // converged for the .aligned TMEM loads
        tc_fence_after();
        const int f = (mt0 + mt) * PF_BM + q * 32 + (lane & ~1);  // first feature of this lane's pair
        const uint32_t ta0 = tmem + buf * C::ACC_COLS + ((uint32_t)(q * 32) << 16);
        const int step = 16 * nparts;
        uint32_t g[16], u[16];
        int c0 = 16 * part;
        if (c0 < npad) {
            tmem_ld16(ta0 + c0, g);
            if (MODE == 0) tmem_ld16(ta0 + C::MAT_COLS + c0, u);
        }
        for (; c0 < npad; c0 += step) {
            tmem_ld_wait16(g);
            if (MODE == 0) reg_tie16(u);
            float o[16];
            if (MODE == 0) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float x = __uint_as_float(g[j]);
                    o[j] = __fdividef(x, 1.0f + __expf(-x)) * __uint_as_float(u[j]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const float4 w4 = *reinterpret_cast<const float4*>(s_w + c0 + j);  // rows past nrows: unused
                    o[j] = w4.x * __uint_as_float(g[j]);
                    o[j + 1] = w4.y * __uint_as_float(g[j + 1]);
                    o[j + 2] = w4.z * __uint_as_float(g[j + 2]);
                    o[j + 3] = w4.w * __uint_as_float(g[j + 3]);
                }
            }
            if (c0 + step < npad) {  // the next chunk loads while this one is stored
                tmem_ld16(ta0 + c0 + step, g);
                if (MODE == 0) tmem_ld16(ta0 + C::MAT_COLS + c0 + step, u);
            }
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
                const float recv = __shfl_xor_sync(0xffffffffu, odd ? o[j] : o[j + 1], 1);
                const uint32_t pk = odd ? pack_bf16x2(recv, o[j + 1]) : pack_bf16x2(o[j], recv);
                const int n = c0 + j + odd;
                if (n < nrows) *reinterpret_cast<uint32_t*>(a.out + (size_t)(row0 + n) * NOUT + f) = pk;
            }
        }
        tc_fence_before();
        __syncwarp();
        if (arrive && lane == 0) mbar_arrive(&acce[buf]);
        return true;
    };

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tx128);
            tma_prefetch_desc(&tx64);
            tma_prefetch_desc(&tx32);
            tma_prefetch_desc(&tx16);
            const uint32_t bytes = npad * PF_BK * 2;
            int s = 0, ph = 0, kb = 0;
            for (int i = 0; i < nstage; ++i) {
                const int kc = kb * PF_BK;
                if (!mbar_wait_fast(&empty[s], ph ^ 1)) break;
                mbar_arrive_expect_tx(&full[s], bytes);
                uint8_t* dst = sB + s * C::B_BYTES;  // row r at r * 128 B
                int r = 0;
                for (; r + 128 <= npad; r += 128) tma_load_2d(dst + r * 128, &tx128, &full[s], kc, row0 + r);
                if (r + 64 <= npad) {
                    tma_load_2d(dst + r * 128, &tx64, &full[s], kc, row0 + r);
                    r += 64;
                }
                if (r + 32 <= npad) {
                    tma_load_2d(dst + r * 128, &tx32, &full[s], kc, row0 + r);
                    r += 32;
                }
                if (r + 16 <= npad) tma_load_2d(dst + r * 128, &tx16, &full[s], kc, row0 + r);
                if (++s == C::TSTAGES) { s = 0; ph ^= 1; }
                if (++kb == nk) kb = 0;
            }
        }
    } else if (warp == 1 || warp == PF_MMA2_WARP) {
        // MMA issue for matrix m (GEMM1: warp 1 gate, warp 22 up; GEMM2: warp 1)
        const int m = warp == 1 ? 0 : 1;
        if (lane == 0 && m < C::NISSUE) {
            // The issuing thread shares its SM sub-partition with four busy
            // dequant warps, so its loop is kept short: ring positions advance
            // incrementally and the B descriptors are offsets of one base (the
            // whole ring lies below 256 KB, inside the descriptor's 14-bit
            // address field, so the additions cannot carry out of it).
            const uint32_t idesc = make_idesc_bf16(PF_BM, npad);
            uint64_t* mdeq = deq + m * C::ASLOTS;
            uint64_t* maempty = aempty + m * C::ASLOTS;
            const uint64_t bdesc0 = make_sdesc_sw128(smem_u32(sB));
            const uint32_t abase = tmem + C::A_COL0 + m * (PF_BK / 2);
            int s = 0, ph = 0, sl = 0, pa = 0;
            for (int mt = 0; mt < nmt && alive; ++mt) {
                const int buf = mt % C::NACC, use = mt / C::NACC;
                if (!mbar_wait_fast(&acce[buf], (use & 1) ^ 1)) { alive = false; break; }  // drained by the epilogue
                tc_fence_after();
                const uint32_t dcol = tmem + buf * C::ACC_COLS + m * C::MAT_COLS;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_fast(&full[s], ph) || !mbar_wait_fast(&mdeq[sl], pa)) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bd = bdesc0 + (uint32_t)(s * (C::B_BYTES >> 4));
                    const uint32_t ac = abase + sl * C::SLOT_COLS;
                    tc_mma_bf16_ts(dcol, ac, bd, idesc, kb != 0);
                    tc_mma_bf16_ts(dcol, ac + 8, bd + 2, idesc, 1u);   // K 16..31: +32 bytes
                    tc_mma_bf16_ts(dcol, ac + 16, bd + 4, idesc, 1u);
                    tc_mma_bf16_ts(dcol, ac + 24, bd + 6, idesc, 1u);
                    tc_commit(&maempty[sl]);  // the A slot may be rewritten
                    tc_commit(&empty[s]);     // this matrix is done with the activation tile
                    if (++s == C::TSTAGES) { s = 0; ph ^= 1; }
                    if (++sl == C::ASLOTS) { sl = 0; pa ^= 1; }
                }
                tc_commit(&accf[buf]);
            }
        }
    } else if (warp >= PF_DQ_WARP0 && warp < PF_DQ_WARP0 + PF_DQ_THREADS / 32) {
        // Warp (quadrant q, group g) owns weight rows 32 q .. 32 q + 31 of the
        // M-tile, one row per lane (its TMEM lane), and one 32-element block of
        // them per stage it takes.  GEMM1: group g = (matrix g / 2, half g % 2)
        // of every stage.  GEMM2: half g % 2 of every other stage (parity g / 2).
        const int q = warp & 3, grp = (warp - PF_DQ_WARP0) >> 2;
        const int m = MODE == 0 ? grp >> 1 : 0;       // matrix
        const int half = grp & 1;                     // block of the stage
        const int i0 = MODE == 0 ? 0 : grp >> 1;      // first stage taken
        constexpr int STRIDE = MODE == 0 ? 1 : 2;     // stages between the ones taken
        uint64_t* mdeq = deq + m * C::ASLOTS;
        uint64_t* maempty = aempty + m * C::ASLOTS;
        const int row = q * 32 + lane;
        const uint8_t* sbase = a.arena + slot * a.slot_bytes;
        const int mi = MODE == 0 ? m : 2;             // arena matrix index
        const uint8_t* cb = sbase + a.off_codes[mi];
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(sbase + a.off_scales[mi]);
        const int bits = MODE == 0 ? (m == 0 ? B0 : B1) : B0;
        const int nb = K / 32;  // blocks (and scales) per weight row
        const uint32_t tcol = tmem + ((uint32_t)(q * 32) << 16) + C::A_COL0 + m * (PF_BK / 2) + half * 16;
        const int ntake = nstage > i0 ? (nstage - i0 + STRIDE - 1) / STRIDE : 0;  // stages this warp takes
        struct Pre {
            uint4 c;
            float s;
        };
        auto fetch = [&](int t, Pre& p) {  // t-th stage taken
            if (t >= ntake) return;
            const int i = i0 + t * STRIDE, mt = i / nk;
            const size_t blk = ((size_t)(mt0 + mt) * PF_BM + row) * nb + 2 * (i - mt * nk) + half;
            p.c = bits == 4 ? load_block_codes<4>(cb + blk * 16) : load_block_codes<2>(cb + blk * 8);
            p.s = half_bits_to_f32(__ldg(sc + blk));
        };
        auto step = [&](int t, const Pre& p) -> bool {
            const int i = i0 + t * STRIDE, sl = i % C::ASLOTS;
            if (!mbar_wait_fast(&maempty[sl], ((i / C::ASLOTS) & 1) ^ 1)) return false;
            tc_fence_after();
            uint32_t col[16];
            if (bits == 4) dequant_block_cols<4>(p.c, p.s, col);
            else dequant_block_cols<2>(p.c, p.s, col);
            tmem_st16(tcol + sl * C::SLOT_COLS, col);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&mdeq[sl]);
            return true;
        };
        static_assert(PF_PREFETCH == 4, "the loop below holds four stages in p0..p3");
        Pre p0{}, p1{}, p2{}, p3{};
        fetch(0, p0);
        fetch(1, p1);
        fetch(2, p2);
        fetch(3, p3);
        bool ok = true;
        for (int t = 0; t < ntake; t += 4) {
            if (!(ok = step(t, p0))) break;
            fetch(t + 4, p0);
            if (t + 1 >= ntake || !(ok = step(t + 1, p1))) break;
            fetch(t + 5, p1);
            if (t + 2 >= ntake || !(ok = step(t + 2, p2))) break;
            fetch(t + 6, p2);
            if (t + 3 >= ntake || !(ok = step(t + 3, p3))) break;
            fetch(t + 7, p3);
        }
        if (ok) drain(nmt - 1, 1 + grp, C::TAIL_DRAIN_PARTS, false);  // the CTA's tail
    } else if (warp >= PF_EPI_WARP0 && warp < PF_EPI_WARP0 + 4) {
        // epilogue warps: part 0 of every M-tile's drain
        for (int mt = 0; mt < nmt && alive; ++mt)
            alive = drain(mt, 0, mt == nmt - 1 ? C::TAIL_DRAIN_PARTS : 1, true);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// Xp[pos][:] = x[perm[pos] / k][:]  (gathered activation rows, bf16).  One warp
// per row, 8 rows per block; a lane's 16-byte loads are all issued before its
// stores.
#define GATHER_ROWS 8
__global__ void __launch_bounds__(32 * GATHER_ROWS) k_gather_rows(const uint16_t* __restrict__ x,
                                                                  const int32_t* __restrict__ perm, int P, int H,
                                                                  int k, uint16_t* __restrict__ xp) {
    const int pos = blockIdx.x * GATHER_ROWS + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (pos >= P) return;
    const int t = perm[pos] / k;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)pos * H);
    const int n = H / 8;  // 16-byte chunks per row
    for (int i0 = lane; i0 < n; i0 += 32 * 8) {
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (i0 + 32 * j < n) v[j] = __ldg(src + i0 + 32 * j);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (i0 + 32 * j < n) dst[i0 + 32 * j] = v[j];
    }
}

