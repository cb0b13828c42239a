// Prefill path: per-expert grouped GEMMs on the 5th-generation tensor cores.
//
// Rows of the grouped activation matrix follow the expert-sorted pair order
// (perm).  A tile is (expert e, up to 256 consecutive pair rows of e, 128
// output features).  The MMA runs "weights x activations": the 128 weight rows
// are the M side, the tile's pair rows the N side (N = rows rounded up to 16),
// so a lightly loaded expert wastes at most 15 columns.
//
//   GEMM1: D_g = W_g[rows] X^T, D_u = W_u[rows] X^T   (K = H)
//          h[pair][row] = bf16(silu(D_g) * D_u)
//   GEMM2: D = W_d[rows] h^T                           (K = I)
//          Y[pair][row] = bf16(w_pair * D)
//
// A CTA owns one N-tile and walks all M-tiles, so the activation rows stay in
// L2 and setup is paid once.  Roles (448 threads): warp 0 issues TMA loads of
// the activation tile (128-B swizzled) and of the raw code tile of each weight
// matrix (one 3-D tensor map spans all arena slots); warp 1 owns TMEM and one
// of its threads issues tcgen05.mma; warps 2-5 drain finished accumulators
// (TMEM -> registers -> global; the down GEMM double-buffers them so this
// overlaps the next M-tile); warps 6-13 dequantise codes to bf16 straight into
// the 128-B swizzled K-major layout the MMA reads.  Stages cycle through full /
// dequantised / empty mbarriers; every wait is bounded.
#pragma once
#include "common.cuh"

#define PF_BK 64          // K elements per stage (one 128-byte swizzle row of bf16)
#define PF_BM 128         // weight rows per M-tile
#define PF_BN_MAX 256     // pair rows per tile (PREFILL_TILE_N)
#define PF_BOX_ROWS 16    // activation rows per TMA box
#define PF_EPI_WARP0 2    // epilogue warps 2..5 (TMEM lane quadrants 2, 3, 0, 1)
#define PF_DQ_WARP0 6     // dequantisation warps 6..13
#define PF_DQ_THREADS 256
#define PF_THREADS 448

template <int MODE>  // 0 = gate/up + SwiGLU, 1 = down + gate weight
struct PfCfg {
    static constexpr int NMAT = MODE == 0 ? 2 : 1;
    static constexpr int TSTAGES = MODE == 0 ? 4 : 5;            // TMA ring: activation tile + raw codes
    static constexpr int ASTAGES = 2;                            // ring of dequantised A tiles
    static constexpr int NACC = MODE == 0 ? 1 : 2;               // accumulator buffers in TMEM
    static constexpr int MAT_COLS = PF_BN_MAX;                   // TMEM columns of one matrix's accumulator
    static constexpr int ACC_COLS = NMAT * PF_BN_MAX;            // TMEM columns of one accumulator buffer
    static constexpr int A_BYTES = PF_BM * PF_BK * 2;            // one dequantised matrix tile
    static constexpr int B_BYTES = PF_BN_MAX * PF_BK * 2;        // activation tile
    static constexpr int C_BYTES = PF_BM * PF_BK / 2;            // raw codes (<= 4-bit)
    static constexpr int SMEM = TSTAGES * (B_BYTES + NMAT * C_BYTES) + ASTAGES * NMAT * A_BYTES +
                                1024 /*align*/ + 1024 /*gate weights*/ + 256 /*barriers*/;
    static constexpr int TMEM_COLS = 512;
};

struct PrefillArgs {
    const uint8_t* arena;
    const int32_t* slot_table;
    int64_t n_slots;
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

// One 32-element block of one row: codes from the staging tile -> 4 swizzled
// 16-byte chunks of the A tile (row r at r * 128 B, chunk j at (j ^ (r & 7)) * 16).
template <int BITS>
__device__ __forceinline__ void dequant_unit(const uint8_t* ctile, uint8_t* atile, int row, int half, float s) {
    constexpr int ROWB = PF_BK * BITS / 8;  // staged code bytes per row
    const uint8_t* src = ctile + row * ROWB + half * (32 * BITS / 8);
    uint32_t w[4];
    if (BITS == 4) {
        uint4 v = *reinterpret_cast<const uint4*>(src);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
        uint2 v = *reinterpret_cast<const uint2*>(src);
        w[0] = v.x & 0xffffu; w[1] = v.x >> 16; w[2] = v.y & 0xffffu; w[3] = v.y >> 16;
    }
    const float shi = __bfloat162float(__float2bfloat16_rn(s));
    const uint32_t s2hi = pack_bf16x2(shi, shi), s2lo = pack_bf16x2(s - shi, s - shi);  // both exact
    uint8_t* rowp = atile + row * 128;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {  // chunk cc holds elements 8cc..8cc+7 of this block
        const int j = half * 4 + cc;
        *reinterpret_cast<uint4*>(rowp + ((j ^ (row & 7)) << 4)) = dq8<BITS>(w[cc], s2hi, s2lo);
    }
}

// One CTA per N-tile (expert e, rows row0 .. row0+nrows of the grouped
// activations); it walks every M-tile of the output features.  Stage i covers
// (M-tile i / nk, K-block i % nk).
template <int MODE, int B0, int B1>
__global__ void __launch_bounds__(PF_THREADS, 1)
    k_prefill_gemm(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC0,
                   const __grid_constant__ CUtensorMap tmC1, PrefillArgs a) {
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
    uint8_t* sB = smem;                                          // [TSTAGES][B_BYTES]
    uint8_t* sC = sB + C::TSTAGES * C::B_BYTES;                  // [TSTAGES][NMAT][C_BYTES]
    uint8_t* sA = sC + C::TSTAGES * C::NMAT * C::C_BYTES;        // [ASTAGES][NMAT][A_BYTES]
    float* s_w = reinterpret_cast<float*>(sA + C::ASTAGES * C::NMAT * C::A_BYTES);  // [PF_BN_MAX] gate weights
    uint64_t* bars = reinterpret_cast<uint64_t*>(s_w + PF_BN_MAX);
    uint64_t* full = bars;                      // [TSTAGES] TMA bytes landed
    uint64_t* empty = full + C::TSTAGES;        // [TSTAGES] codes dequantised and activation tile consumed
    uint64_t* deq = empty + C::TSTAGES;         // [ASTAGES] dequantised A written
    uint64_t* aempty = deq + C::ASTAGES;        // [ASTAGES] MMA finished reading the A tile
    uint64_t* accf = aempty + C::ASTAGES;       // [NACC] accumulator final
    uint64_t* acce = accf + C::NACC;            // [NACC] accumulator drained
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + C::NACC);

    const int64_t slot = a.slot_table[(int64_t)a.layer * a.E + e];
    if (slot < 0 || slot >= a.n_slots) {  // expert without weights contributes zero
        if (threadIdx.x == 0) moe_set_status(MOE_ERR_SLOT);
        for (int i = threadIdx.x; i < nrows * NOUT; i += blockDim.x)
            a.out[(size_t)(row0 + i / NOUT) * NOUT + i % NOUT] = 0;
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::TSTAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], PF_DQ_THREADS / 32 + 1);  // every dequant warp, and the MMA commit
        }
        for (int s = 0; s < C::ASTAGES; ++s) {
            mbar_init(&deq[s], PF_DQ_THREADS / 32);
            mbar_init(&aempty[s], 1);
        }
        for (int b = 0; b < C::NACC; ++b) {
            mbar_init(&accf[b], 1);
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

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tmB);
            tma_prefetch_desc(&tmC0);
            if (C::NMAT == 2) tma_prefetch_desc(&tmC1);
            const uint32_t bytes = npad * PF_BK * 2 + PF_BM * PF_BK * B0 / 8 + (C::NMAT == 2 ? PF_BM * PF_BK * B1 / 8 : 0);
            for (int i = 0; i < nstage && alive; ++i) {
                const int s = i % C::TSTAGES, ph = (i / C::TSTAGES) & 1;
                const int kb = i % nk, rowbase = (mt0 + i / nk) * PF_BM;
                if (!mbar_wait(&empty[s], ph ^ 1)) { alive = false; break; }
                mbar_arrive_expect_tx(&full[s], bytes);
                for (int r = 0; r < npad; r += PF_BOX_ROWS)
                    tma_load_2d(sB + s * C::B_BYTES + r * 128, &tmB, &full[s], kb * PF_BK, row0 + r);
                asm volatile(
                    "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
                        "r"(smem_u32(sC + (s * C::NMAT + 0) * C::C_BYTES)), "l"(&tmC0), "r"(smem_u32(&full[s])),
                    "r"(kb * PF_BK * B0 / 8), "r"(rowbase), "r"((int)slot)
                    : "memory");
                if (C::NMAT == 2)
                    asm volatile(
                        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
                            "r"(smem_u32(sC + (s * C::NMAT + 1) * C::C_BYTES)), "l"(&tmC1), "r"(smem_u32(&full[s])),
                        "r"(kb * PF_BK * B1 / 8), "r"(rowbase), "r"((int)slot)
                        : "memory");
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(PF_BM, npad);
            for (int mt = 0; mt < nmt && alive; ++mt) {
                const int buf = mt % C::NACC, use = mt / C::NACC;
                if (!mbar_wait(&acce[buf], (use & 1) ^ 1)) { alive = false; break; }  // drained by the epilogue
                tc_fence_after();
                const uint32_t dcol = tmem + buf * C::ACC_COLS;
                for (int kb = 0; kb < nk; ++kb) {
                    const int i = mt * nk + kb;
                    const int s = i % C::TSTAGES, ph = (i / C::TSTAGES) & 1;
                    const int sa = i % C::ASTAGES, pa = (i / C::ASTAGES) & 1;
                    if (!mbar_wait(&full[s], ph) || !mbar_wait(&deq[sa], pa)) { alive = false; break; }
                    tc_fence_after();
                    const uint32_t bb = smem_u32(sB + s * C::B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < PF_BK / 16; ++kk) {
                        const uint64_t bdesc = make_sdesc_sw128(bb + kk * 32);
#pragma unroll
                        for (int m = 0; m < C::NMAT; ++m) {
                            const uint32_t ab = smem_u32(sA + (sa * C::NMAT + m) * C::A_BYTES);
                            tc_mma_bf16(dcol + m * C::MAT_COLS, make_sdesc_sw128(ab + kk * 32), bdesc, idesc,
                                        (kb | kk) != 0);
                        }
                    }
                    tc_commit(&empty[s]);    // the activation tile may be refilled
                    tc_commit(&aempty[sa]);  // the A tile may be rewritten
                }
                tc_commit(&accf[buf]);
            }
        }
    } else if (warp >= PF_DQ_WARP0) {
        const int dt = threadIdx.x - PF_DQ_WARP0 * 32;  // 0..255
        const int row = dt >> 1, half = dt & 1;
        const uint8_t* sbase = a.arena + slot * a.slot_bytes;
        const uint16_t* sc0 = reinterpret_cast<const uint16_t*>(sbase + a.off_scales[MODE == 0 ? 0 : 2]);
        const uint16_t* sc1 = reinterpret_cast<const uint16_t*>(sbase + a.off_scales[1]);
        // One 16-byte load holds this thread's scales for 4 consecutive stages (blocks
        // 2 kb .. 2 kb + 7 of its row); when nk % 4 == 0 groups of 4 stages never
        // straddle an M-tile and the next group's scales are loaded a group ahead.
        // Otherwise (K % 256 != 0) each stage loads its own scale.
        const bool grouped = (nk & 3) == 0;
        const int ngrp = grouped ? nstage / 4 : 0;
        auto load_grp = [&](int gi, uint4& r0, uint4& r1) {
            const int i0 = gi * 4, kb0 = i0 % nk;
            const size_t base = (size_t)((mt0 + i0 / nk) * PF_BM + row) * (K / 32) + 2 * kb0;
            r0 = __ldg(reinterpret_cast<const uint4*>(sc0 + base));
            if (C::NMAT == 2) r1 = __ldg(reinterpret_cast<const uint4*>(sc1 + base));
        };
        auto pick = [](const uint4& v, int idx) -> uint16_t {  // half idx (0..7) of v
            const int wi = idx >> 1;
            const uint32_t w = wi == 0 ? v.x : (wi == 1 ? v.y : (wi == 2 ? v.z : v.w));
            return (uint16_t)(w >> (16 * (idx & 1)));
        };
        uint4 cur0 = make_uint4(0, 0, 0, 0), cur1 = cur0, nxt0 = cur0, nxt1 = cur0;
        if (ngrp > 0) load_grp(0, cur0, cur1);
        if (ngrp > 1) load_grp(1, nxt0, nxt1);
        for (int i = 0; i < nstage; ++i) {
            const int s = i % C::TSTAGES, ph = (i / C::TSTAGES) & 1;
            const int sa = i % C::ASTAGES, pa = (i / C::ASTAGES) & 1;
            uint16_t q0, q1 = 0;
            if (grouped) {
                if ((i & 3) == 0 && i > 0) {
                    cur0 = nxt0;
                    cur1 = nxt1;
                    if ((i >> 2) + 1 < ngrp) load_grp((i >> 2) + 1, nxt0, nxt1);
                }
                const int si = 2 * (i & 3) + half;
                q0 = pick(cur0, si);
                if (C::NMAT == 2) q1 = pick(cur1, si);
            } else {
                const size_t grow = (size_t)((mt0 + i / nk) * PF_BM + row);  // weight row in the matrix
                q0 = __ldg(sc0 + grow * (K / 32) + 2 * (i % nk) + half);
                if (C::NMAT == 2) q1 = __ldg(sc1 + grow * (K / 32) + 2 * (i % nk) + half);
            }
            if (!mbar_wait(&full[s], ph) || !mbar_wait(&aempty[sa], pa ^ 1)) { alive = false; break; }
            dequant_unit<B0>(sC + (s * C::NMAT + 0) * C::C_BYTES, sA + (sa * C::NMAT + 0) * C::A_BYTES, row, half,
                             half_bits_to_f32(q0));
            if (C::NMAT == 2)
                dequant_unit<B1>(sC + (s * C::NMAT + 1) * C::C_BYTES, sA + (sa * C::NMAT + 1) * C::A_BYTES, row,
                                 half, half_bits_to_f32(q1));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&deq[sa]);
                mbar_arrive(&empty[s]);  // this warp's reads of the codes are done
            }
        }
    } else {  // epilogue warps: TMEM -> registers -> global, one M-tile at a time
        const int q = warp & 3;  // TMEM lane quadrant this warp may read
        for (int mt = 0; mt < nmt && alive; ++mt) {
            const int buf = mt % C::NACC, use = mt / C::NACC;
            if (!mbar_wait(&accf[buf], use & 1)) { alive = false; break; }
            tc_fence_after();
            const int r = (mt0 + mt) * PF_BM + q * 32 + lane;  // output feature of this thread
            const uint32_t ta0 = tmem + buf * C::ACC_COLS + ((uint32_t)(q * 32) << 16);
            for (int c0 = 0; c0 < npad; c0 += 16) {
                uint32_t v0[16], v1[16];
                tmem_ld16(ta0 + c0, v0);
                if (MODE == 0) tmem_ld16(ta0 + C::MAT_COLS + c0, v1);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int n = c0 + j;
                    if (n < nrows) {
                        float o;
                        if (MODE == 0) o = silu_f32(__uint_as_float(v0[j])) * __uint_as_float(v1[j]);
                        else o = s_w[n] * __uint_as_float(v0[j]);
                        a.out[(size_t)(row0 + n) * NOUT + r] = f32_to_bf16_bits(o);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[buf]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// Xp[pos][:] = x[perm[pos] / k][:]  (gathered activation rows, bf16)
__global__ void k_gather_rows(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, int P, int H, int k,
                              uint16_t* __restrict__ xp) {
    const int pos = blockIdx.x;
    if (pos >= P) return;
    const int t = perm[pos] / k;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)pos * H);
    for (int i = threadIdx.x; i < H / 8; i += blockDim.x) dst[i] = __ldg(src + i);
}
