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
// Roles (384 threads): warp 0 issues TMA loads of the activation tile (128-B
// swizzled) and of the raw code tile of each weight matrix; warp 1 owns TMEM
// and one of its threads issues tcgen05.mma; warps 4-11 dequantise codes to
// bf16 straight into the 128-B swizzled K-major layout the MMA reads, then run
// the epilogue from TMEM.  Stages cycle through full / dequantised / empty
// mbarriers; every wait is bounded.
#pragma once
#include "common.cuh"

#define PF_BK 64          // K elements per stage (one 128-byte swizzle row of bf16)
#define PF_BM 128         // weight rows per tile
#define PF_BN_MAX 256     // pair rows per tile
#define PF_BOX_ROWS 16    // activation rows per TMA box
#define PF_THREADS 384
#define PF_DQ_WARP0 4     // first dequant / epilogue warp
#define PF_DQ_THREADS 256

template <int MODE>  // 0 = gate/up + SwiGLU, 1 = down + gate weight
struct PfCfg {
    static constexpr int NMAT = MODE == 0 ? 2 : 1;
    static constexpr int STAGES = MODE == 0 ? 3 : 4;
    static constexpr int A_BYTES = PF_BM * PF_BK * 2;            // one dequantised matrix tile
    static constexpr int B_BYTES = PF_BN_MAX * PF_BK * 2;        // activation tile
    static constexpr int C_BYTES = PF_BM * PF_BK / 2;            // raw codes (<= 4-bit)
    static constexpr int STAGE_BYTES = NMAT * A_BYTES + B_BYTES + NMAT * C_BYTES;
    static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
    static constexpr int TMEM_COLS = MODE == 0 ? 512 : 256;
};

struct PrefillArgs {
    const uint8_t* arena;
    const int32_t* slot_table;
    int64_t n_slots;
    int64_t off_scales[3];
    int64_t slot_bytes;
    int H, I, E, k, layer;
    const int4* tiles;       // (expert, first pair row, rows, 0)
    const int32_t* meta;     // [1] = number of tiles
    const int32_t* perm;
    const float* topk_w;
    uint16_t* out;           // GEMM1: h [P][I]; GEMM2: Y [P][H]
};

// codes of 8 consecutive 4-bit (or 2-bit) elements -> 8 dequantised bf16 (uint4)
template <int BITS>
__device__ __forceinline__ uint4 dq8(uint32_t w, float s) {
    constexpr float kMagic = 8388608.0f + (float)(1 << (BITS - 1));  // 2^23 + offset
    float f[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t q = (w >> (BITS * i)) & ((1u << BITS) - 1);
        f[i] = (__uint_as_float(0x4B000000u | q) - kMagic) * s;  // exact (q - offset) * s, one rounding
    }
    uint4 r;
    r.x = pack_bf16x2(f[0], f[1]);
    r.y = pack_bf16x2(f[2], f[3]);
    r.z = pack_bf16x2(f[4], f[5]);
    r.w = pack_bf16x2(f[6], f[7]);
    return r;
}

// One 32-element block of one row: codes from the staging tile -> 4 swizzled
// 16-byte chunks of the A tile.
template <int BITS>
__device__ __forceinline__ void dequant_unit(const uint8_t* ctile, uint8_t* atile, int row, int half, float s) {
    constexpr int ROWB = PF_BK * BITS / 8;  // staged code bytes per row
    const uint8_t* src = ctile + row * ROWB + half * (32 * BITS / 8);
    uint32_t w[BITS];  // 32 codes = BITS words
    if (BITS == 4) {
        uint4 v = *reinterpret_cast<const uint4*>(src);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
        uint2 v = *reinterpret_cast<const uint2*>(src);
        w[0] = v.x; w[1] = v.y;
    }
    uint8_t* rowp = atile + row * 128;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
        // chunk cc holds elements 8cc..8cc+7 of this block
        uint32_t codes = (BITS == 4) ? w[cc] : ((w[cc >> 1] >> (16 * (cc & 1))) & 0xffffu);
        uint4 v = dq8<BITS>(codes, s);
        int j = half * 4 + cc;
        *reinterpret_cast<uint4*>(rowp + ((j ^ (row & 7)) << 4)) = v;
    }
}

template <int MODE, int B0, int B1>
__global__ void __launch_bounds__(PF_THREADS, 1)
    k_prefill_gemm(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC0,
                   const __grid_constant__ CUtensorMap tmC1, PrefillArgs a) {
    using C = PfCfg<MODE>;
    const int tile = blockIdx.y;
    if (tile >= a.meta[1]) return;
    const int4 td = a.tiles[tile];
    const int e = td.x, row0 = td.y, nrows = td.z;
    const int npad = (nrows + 15) & ~15;
    const int mt = blockIdx.x;
    const int K = MODE == 0 ? a.H : a.I;
    const int NOUT = MODE == 0 ? a.I : a.H;  // output features (row length of `out`)
    const int nk = K / PF_BK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* sB = smem;                                          // [STAGES][B_BYTES]
    uint8_t* sA = sB + C::STAGES * C::B_BYTES;                   // [STAGES][NMAT][A_BYTES]
    uint8_t* sC = sA + C::STAGES * C::NMAT * C::A_BYTES;         // [STAGES][NMAT][C_BYTES]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sC + C::STAGES * C::NMAT * C::C_BYTES);
    uint64_t* full = bars;                   // TMA bytes landed
    uint64_t* deq = bars + C::STAGES;        // dequantised A written
    uint64_t* empty = bars + 2 * C::STAGES;  // MMA finished reading the stage
    uint64_t* accf = bars + 3 * C::STAGES;   // accumulators final
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);

    const int64_t slot = a.slot_table[(int64_t)a.layer * a.E + e];
    if (slot < 0 || slot >= a.n_slots) {  // expert without weights contributes zero
        if (threadIdx.x == 0 && mt == 0) moe_set_status(MOE_ERR_SLOT);
        for (int i = threadIdx.x; i < nrows * PF_BM; i += blockDim.x) {
            int n = i / PF_BM, r = i % PF_BM;
            a.out[(size_t)(row0 + n) * NOUT + mt * PF_BM + r] = 0;
        }
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&deq[s], PF_DQ_THREADS / 32);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        fence_mbar_init();
    }
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
            for (int i = 0; i < nk && alive; ++i) {
                const int s = i % C::STAGES, ph = (i / C::STAGES) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1)) { alive = false; break; }
                mbar_arrive_expect_tx(&full[s], bytes);
                for (int r = 0; r < npad; r += PF_BOX_ROWS)
                    tma_load_2d(sB + s * C::B_BYTES + r * 128, &tmB, &full[s], i * PF_BK, row0 + r);
                const int rowbase = mt * PF_BM;
                asm volatile(
                    "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
                        "r"(smem_u32(sC + (s * C::NMAT + 0) * C::C_BYTES)), "l"(&tmC0), "r"(smem_u32(&full[s])),
                    "r"(i * PF_BK * B0 / 8), "r"(rowbase), "r"((int)slot)
                    : "memory");
                if (C::NMAT == 2)
                    asm volatile(
                        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
                            "r"(smem_u32(sC + (s * C::NMAT + 1) * C::C_BYTES)), "l"(&tmC1), "r"(smem_u32(&full[s])),
                        "r"(i * PF_BK * B1 / 8), "r"(rowbase), "r"((int)slot)
                        : "memory");
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(PF_BM, npad);
            for (int i = 0; i < nk && alive; ++i) {
                const int s = i % C::STAGES, ph = (i / C::STAGES) & 1;
                if (!mbar_wait(&full[s], ph) || !mbar_wait(&deq[s], ph)) { alive = false; break; }
                tc_fence_after();
                const uint32_t bb = smem_u32(sB + s * C::B_BYTES);
#pragma unroll
                for (int kk = 0; kk < PF_BK / 16; ++kk) {
                    const uint64_t bdesc = make_sdesc_sw128(bb + kk * 32);
#pragma unroll
                    for (int m = 0; m < C::NMAT; ++m) {
                        const uint32_t ab = smem_u32(sA + (s * C::NMAT + m) * C::A_BYTES);
                        tc_mma_bf16(tmem + m * 256, make_sdesc_sw128(ab + kk * 32), bdesc, idesc, (i | kk) != 0);
                    }
                }
                tc_commit(&empty[s]);
            }
            tc_commit(accf);
        }
    } else if (warp >= PF_DQ_WARP0) {
        const int dt = threadIdx.x - PF_DQ_WARP0 * 32;  // 0..255
        const int row = dt >> 1, half = dt & 1;
        const int grow = mt * PF_BM + row;  // weight row in the matrix
        const uint16_t* sc0 = reinterpret_cast<const uint16_t*>(a.arena + slot * a.slot_bytes +
                                                               a.off_scales[MODE == 0 ? 0 : 2]) +
                              (size_t)grow * (K / 32);
        const uint16_t* sc1 =
            reinterpret_cast<const uint16_t*>(a.arena + slot * a.slot_bytes + a.off_scales[1]) + (size_t)grow * (K / 32);
        for (int i = 0; i < nk; ++i) {
            const int s = i % C::STAGES, ph = (i / C::STAGES) & 1;
            if (!mbar_wait(&full[s], ph)) { alive = false; break; }
            const float s0 = half_bits_to_f32(__ldg(sc0 + 2 * i + half));
            dequant_unit<B0>(sC + (s * C::NMAT + 0) * C::C_BYTES, sA + (s * C::NMAT + 0) * C::A_BYTES, row, half, s0);
            if (C::NMAT == 2) {
                const float s1 = half_bits_to_f32(__ldg(sc1 + 2 * i + half));
                dequant_unit<B1>(sC + (s * C::NMAT + 1) * C::C_BYTES, sA + (s * C::NMAT + 1) * C::A_BYTES, row, half,
                                 s1);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&deq[s]);
        }
        // epilogue: TMEM -> registers -> global
        if (alive && mbar_wait(accf, 0)) {
            tc_fence_after();
            const int q = warp & 3;              // TMEM lane quadrant this warp may read
            const int chalf = (warp - PF_DQ_WARP0) >> 2;
            const int r = mt * PF_BM + q * 32 + lane;  // output feature of this thread
            for (int c0 = chalf * 16; c0 < npad; c0 += 32) {
                uint32_t v0[16], v1[16];
                const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + c0;
                tmem_ld16(ta, v0);
                if (MODE == 0) tmem_ld16(ta + 256, v1);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int n = c0 + j;
                    if (n < nrows) {
                        float o;
                        if (MODE == 0) {
                            o = silu_f32(__uint_as_float(v0[j])) * __uint_as_float(v1[j]);
                        } else {
                            o = __ldg(a.topk_w + a.perm[row0 + n]) * __uint_as_float(v0[j]);
                        }
                        a.out[(size_t)(row0 + n) * NOUT + r] = f32_to_bf16_bits(o);
                    }
                }
            }
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
