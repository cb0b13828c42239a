// Decode window (T <= 8 tokens) as one persistent, cooperatively launched
// kernel per layer: one CTA per SM, two grid-wide barriers.
//
//   A  router logits in fp64 (warp per expert, experts spread over all SMs)
//   -- barrier --
//   B  every CTA certifies the top-k of every token (the same deterministic
//      computation everywhere, so no second barrier is needed) and builds
//      the grouping (pairs sorted by expert) in shared memory; CTA 0 writes
//      the routing outputs and the histogram
//   C  gate/up + SwiGLU: each CTA owns a contiguous range of 16-row tiles of
//      the selected experts; codes and scales stream through a ring of TMA
//      stages; the dot products run on mma.sync m16n8k16 (bf16 in, fp32 out)
//      with all T tokens as the 8 columns, so the cost per weight is the
//      unpack alone; W_d rows needed in D are prefetched into L2
//   -- barrier --
//   D  down + combine: each CTA owns 16 output features for every selected
//      expert, so it holds complete sums and writes out[t][f] directly, in
//      a fixed slot order.
//
// Codes enter the MMA as (128 + q) in bf16 (an exponent-bias bit pattern:
// 0x4300 | q), so each block's MMA result is sum q x + 128 sum x; the block
// correction (128 + offset) * sum x is subtracted and the block scale applied
// in fp32.  All waits (ring mbarriers, grid barriers) are bounded.
#pragma once
#include "common.cuh"
#include "perm.cuh"
#include "router.cuh"

#define DF_WARPS 16
#define DF_THREADS (32 * DF_WARPS)
#define DF_STAGES 6
#define DF_SLOT 20480
#define DF_TN 8          // token columns of the MMA
#define DF_MAXP 256      // pairs T * k
#define DF_FT 16         // features per CTA in phase D

struct DecodeFusedArgs {
    const uint8_t* arena;
    const int32_t* slot_table;
    int64_t n_slots;
    int64_t off_codes[3], off_scales[3];
    int64_t slot_bytes;
    int H, I, E, k, layer, T, residual;
    int bits_g, bits_u, bits_d;
    int chunk;               // gate/up K-chunk (elements)
    const uint16_t* x;       // [T][H]
    const float* W;          // router [E][H]
    const float* b;          // router bias [E] or null
    uint16_t* out;           // [T][H]
    uint32_t* hist;          // [L][E] or null
    int32_t* idx;            // [T*k]
    float* w;                // [T*k]
    int32_t* offsets;        // [E+1]
    int32_t* perm;           // [T*k]
    int32_t* nrechk;         // [1]
    double* logit;           // [T][E] workspace
    double* absum;           // [T][E] workspace
    uint16_t* hB;            // [P][I] bf16, MMA-fragment order within each 32-block
    float* hC;               // [P][I/16] sums of h over 16-row halves of each block
    unsigned int* bar;       // grid barrier counter (zeroed before launch)
};

// ---------------------------------------------------------------- small helpers

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier over `nblocks` co-resident CTAs; the counter only grows
// (target = nblocks * phase).  Bounded: on expiry the status word gets
// MOE_ERR_TIMEOUT and every thread of the CTA sees false.
__device__ __forceinline__ bool grid_barrier(unsigned* ctr, unsigned target, int site) {
    __syncthreads();
    int ok = 1;
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(ctr, 1u);
        unsigned it = 0;
        while (ld_acquire_u32(ctr) < target) {
            if (++it > MOE_SPIN_LIMIT) { moe_note_timeout(site, (int)(ld_acquire_u32(ctr) % 1000)); ok = 0; break; }
            if (it > 32) __nanosleep(64);
        }
        __threadfence();
    }
    return __syncthreads_and(ok) != 0;
}

// Bounded wait until the producer has started unit i in ring slot s.
__device__ __forceinline__ bool wait_slot(volatile int* slot_seq, int s, int i, int site) {
    for (uint32_t it = 0; it < MOE_SPIN_LIMIT; ++it) {
        if (slot_seq[s] == i) return true;
        if (it > 32) __nanosleep(64);
    }
    moe_note_timeout(site, i);
    return false;
}

// bf16 pairs (128 + q_i, 128 + q_{i+4}) of 8 codes: 4-bit word w = codes
// 0..7 in nibbles; 2-bit: codes 0..7 in the low 16 bits.
template <int BITS>
__device__ __forceinline__ void unpack8(uint32_t w, uint32_t (&p)[4]) {
    if (BITS == 4) {
        p[0] = (w & 0x000F000Fu) | 0x43004300u;
        p[1] = ((w >> 4) & 0x000F000Fu) | 0x43004300u;
        p[2] = ((w >> 8) & 0x000F000Fu) | 0x43004300u;
        p[3] = ((w >> 12) & 0x000F000Fu) | 0x43004300u;
    } else {
        const uint32_t v = __byte_perm(w, 0, 0x4140);  // byte0 -> byte 0, byte1 -> byte 2
        p[0] = (v & 0x00030003u) | 0x43004300u;
        p[1] = ((v >> 2) & 0x00030003u) | 0x43004300u;
        p[2] = ((v >> 4) & 0x00030003u) | 0x43004300u;
        p[3] = ((v >> 6) & 0x00030003u) | 0x43004300u;
    }
}

// D(4 fp32) = A(16x16 bf16) * B(16x8 bf16), accumulator starting at zero
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Word q (8 codes) of quant block j of row r in a 16-row code tile staged by
// TMA with 128-byte swizzle (16 rows x 128 B per box, boxes stacked along K).
template <int BITS>
__device__ __forceinline__ uint32_t tile_word(const uint8_t* tile, int r, int j, int q) {
    constexpr int BLK_B = 32 * BITS / 8;      // bytes per quant block
    constexpr int PER_BOX = 128 / BLK_B;      // blocks per 128-byte box row
    const int box = j / PER_BOX, off = (j % PER_BOX) * BLK_B + q * BITS;  // byte offset in the row
    const uint8_t* p = tile + box * 2048 + r * 128 + ((((off >> 4) ^ (r & 7)) << 4) | (off & 15));
    if (BITS == 4) return *reinterpret_cast<const uint32_t*>(p);
    return *reinterpret_cast<const uint16_t*>(p);
}

// 8 bf16 of a row in the fragment order used for B: elements (0,4),(1,5),(2,6),(3,7)
__device__ __forceinline__ uint4 frag_order8(const float (&v)[8]) {
    uint4 r;
    r.x = pack_bf16x2(v[0], v[4]);
    r.y = pack_bf16x2(v[1], v[5]);
    r.z = pack_bf16x2(v[2], v[6]);
    r.w = pack_bf16x2(v[3], v[7]);
    return r;
}

// ---------------------------------------------------------------- shared memory plan

struct DfRoute {  // grouping of the window's pairs, identical in every CTA
    int32_t idx[DF_MAXP];   // expert of pair p = t*k + j
    float w[DF_MAXP];
    int32_t perm[DF_MAXP];  // position -> pair
    int32_t inv[DF_MAXP];   // pair -> position
    int32_t u_e[DF_MAXP];   // selected experts, ascending
    int32_t u_pos[DF_MAXP]; // first position of each
    int32_t u_n[DF_MAXP];   // pairs of each
    int32_t n_uniq;
};

// ---------------------------------------------------------------- phase C: one 16-row tile

// Accumulates gate and up for rows (g, g+8) of the tile and token columns
// (2q, 2q+1) over one K-chunk staged in `slot`.
template <int BG, int BU>
__device__ __forceinline__ void gateup_chunk(const uint8_t* slot, int chunk, int nbox_g, int nbox_u, int j0,
                                             const uint4* xb, const float* xc, float (&accg)[4], float (&accu)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const uint8_t* cg = slot;
    const uint8_t* cu = cg + nbox_g * 2048;
    const uint16_t* sg = reinterpret_cast<const uint16_t*>(cu + nbox_u * 2048);
    const uint16_t* su = sg + 16 * (chunk / 32);
    const int nblk = chunk / 32;
    constexpr float kOffG = 128.f + (float)(1 << (BG - 1)), kOffU = 128.f + (float)(1 << (BU - 1));
#pragma unroll 2
    for (int jj = 0; jj < nblk; ++jj) {
        const int j = j0 + jj;  // block index along H
        const uint4 bx = xb[(j * 4 + q) * DF_TN + g];  // x fragments of token g
        uint32_t pg0[4], pg1[4], pu0[4], pu1[4];
        unpack8<BG>(tile_word<BG>(cg, g, jj, q), pg0);
        unpack8<BG>(tile_word<BG>(cg, g + 8, jj, q), pg1);
        unpack8<BU>(tile_word<BU>(cu, g, jj, q), pu0);
        unpack8<BU>(tile_word<BU>(cu, g + 8, jj, q), pu1);
        float dg[4] = {0.f, 0.f, 0.f, 0.f}, du[4] = {0.f, 0.f, 0.f, 0.f};
        mma_bf16_16816(dg, pg0[0], pg1[0], pg0[1], pg1[1], bx.x, bx.y);
        mma_bf16_16816(dg, pg0[2], pg1[2], pg0[3], pg1[3], bx.z, bx.w);
        mma_bf16_16816(du, pu0[0], pu1[0], pu0[1], pu1[1], bx.x, bx.y);
        mma_bf16_16816(du, pu0[2], pu1[2], pu0[3], pu1[3], bx.z, bx.w);
        const float2 sx = *reinterpret_cast<const float2*>(xc + j * DF_TN + 2 * q);  // sum x, tokens 2q, 2q+1
        const float sg0 = half_bits_to_f32(sg[g * nblk + jj]), sg1 = half_bits_to_f32(sg[(g + 8) * nblk + jj]);
        const float su0 = half_bits_to_f32(su[g * nblk + jj]), su1 = half_bits_to_f32(su[(g + 8) * nblk + jj]);
        accg[0] = fmaf(sg0, fmaf(-kOffG, sx.x, dg[0]), accg[0]);
        accg[1] = fmaf(sg0, fmaf(-kOffG, sx.y, dg[1]), accg[1]);
        accg[2] = fmaf(sg1, fmaf(-kOffG, sx.x, dg[2]), accg[2]);
        accg[3] = fmaf(sg1, fmaf(-kOffG, sx.y, dg[3]), accg[3]);
        accu[0] = fmaf(su0, fmaf(-kOffU, sx.x, du[0]), accu[0]);
        accu[1] = fmaf(su0, fmaf(-kOffU, sx.y, du[1]), accu[1]);
        accu[2] = fmaf(su1, fmaf(-kOffU, sx.x, du[2]), accu[2]);
        accu[3] = fmaf(su1, fmaf(-kOffU, sx.y, du[3]), accu[3]);
    }
}

// ---------------------------------------------------------------- phase D: one expert's 16 features

template <int BD>
__device__ __forceinline__ void down_unit(const DecodeFusedArgs& a, const uint8_t* slot, int nbox, int pos0, int n,
                                          float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int nblk = a.I / 32;
    const uint16_t* sd = reinterpret_cast<const uint16_t*>(slot + nbox * 2048);
    constexpr float kOff = 128.f + (float)(1 << (BD - 1));
    const bool col_ok = g < n;  // B column g = pair pos0 + g
    const uint4* hb = reinterpret_cast<const uint4*>(a.hB + (size_t)(pos0 + (col_ok ? g : 0)) * a.I);
    const float* hc0 = a.hC + (size_t)(pos0 + 2 * q) * (a.I / 16);
    const float* hc1 = a.hC + (size_t)(pos0 + 2 * q + 1) * (a.I / 16);
    const bool c0 = 2 * q < n, c1 = 2 * q + 1 < n;
#pragma unroll 2
    for (int j = 0; j < nblk; ++j) {
        uint4 bx = col_ok ? hb[j * 4 + q] : make_uint4(0, 0, 0, 0);
        uint32_t p0[4], p1[4];
        unpack8<BD>(tile_word<BD>(slot, g, j, q), p0);
        unpack8<BD>(tile_word<BD>(slot, g + 8, j, q), p1);
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        mma_bf16_16816(d, p0[0], p1[0], p0[1], p1[1], bx.x, bx.y);
        mma_bf16_16816(d, p0[2], p1[2], p0[3], p1[3], bx.z, bx.w);
        const float s0 = half_bits_to_f32(sd[g * nblk + j]), s1 = half_bits_to_f32(sd[(g + 8) * nblk + j]);
        const float h0 = c0 ? hc0[2 * j] + hc0[2 * j + 1] : 0.f;
        const float h1 = c1 ? hc1[2 * j] + hc1[2 * j + 1] : 0.f;
        acc[0] = fmaf(s0, fmaf(-kOff, h0, d[0]), acc[0]);
        acc[1] = fmaf(s0, fmaf(-kOff, h1, d[1]), acc[1]);
        acc[2] = fmaf(s1, fmaf(-kOff, h0, d[2]), acc[2]);
        acc[3] = fmaf(s1, fmaf(-kOff, h1, d[3]), acc[3]);
    }
}

// ---------------------------------------------------------------- the kernel

__host__ __device__ constexpr int df_smem_bytes(int H) {
    return 1024 /*align*/ + DF_STAGES * DF_SLOT + H * 16 /*x fragments*/ + (H / 32) * DF_TN * 4 /*block sums*/ +
           DF_MAXP * DF_FT * 4 /*per-pair outputs*/ + (int)sizeof(DfRoute) + 2 * DF_STAGES * 8 + DF_STAGES * 4 + 64;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, uint64_t* bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
            "r"(smem_u32(dst)),
        "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

template <int BG, int BU, int BD>
__global__ void __launch_bounds__(DF_THREADS, 1)
    k_decode_fused(const __grid_constant__ CUtensorMap tcg, const __grid_constant__ CUtensorMap tcu,
                   const __grid_constant__ CUtensorMap tcd, const __grid_constant__ CUtensorMap tsg,
                   const __grid_constant__ CUtensorMap tsu, const __grid_constant__ CUtensorMap tsd,
                   DecodeFusedArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int H = a.H, I = a.I, E = a.E, k = a.k, T = a.T, P = T * k;
    uint4* xb = reinterpret_cast<uint4*>(ring + DF_STAGES * DF_SLOT);  // [H/32][4][8]
    float* xc = reinterpret_cast<float*>(xb + (H / 32) * 4 * DF_TN);     // [H/32][8]
    float* ypair = xc + (H / 32) * DF_TN;                               // [MAXP][FT]
    DfRoute* rt = reinterpret_cast<DfRoute*>(ypair + DF_MAXP * DF_FT);
    uint64_t* full = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(rt + 1) + 7) & ~(uintptr_t)7);
    uint64_t* empty = full + DF_STAGES;
    // slot_seq[s] = the unit the producer last started in slot s.  Several
    // warps consume the ring, so a consumer may reach unit i while unit i - S
    // still owns the slot; a parity wait cannot tell those phases apart, so it
    // first waits for slot_seq[s] == i.
    volatile int* slot_seq = reinterpret_cast<volatile int*>(empty + DF_STAGES);
    __shared__ int s_cnt[MOE_MAX_E];
    __shared__ int s_off[MOE_MAX_E];
    __shared__ int s_warp[33];

    const int G = gridDim.x, cta = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    bool alive = true;

    if (tid == 0) {
        for (int s = 0; s < DF_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            slot_seq[s] = -1;
        }
        fence_mbar_init();
    }
    // x as MMA B fragments (token columns 0..7, zero beyond T) and per-block sums
    for (int u = tid; u < (H / 32) * 4 * DF_TN; u += DF_THREADS) {
        const int n = u % DF_TN, q = (u / DF_TN) % 4, j = u / (DF_TN * 4);
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (n < T) {
            uint4 r = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)n * H + 32 * j + 8 * q));
            v[0] = __uint_as_float(r.x << 16); v[1] = __uint_as_float(r.x & 0xffff0000u);
            v[2] = __uint_as_float(r.y << 16); v[3] = __uint_as_float(r.y & 0xffff0000u);
            v[4] = __uint_as_float(r.z << 16); v[5] = __uint_as_float(r.z & 0xffff0000u);
            v[6] = __uint_as_float(r.w << 16); v[7] = __uint_as_float(r.w & 0xffff0000u);
        }
        xb[u] = frag_order8(v);
    }
    for (int u = tid; u < (H / 32) * DF_TN; u += DF_THREADS) {
        const int n = u % DF_TN, j = u / DF_TN;
        float sx = 0.f;
        if (n < T)
            for (int e = 0; e < 32; ++e) sx += bf16_bits_to_f32(a.x[(size_t)n * H + 32 * j + e]);
        xc[u] = sx;
    }

    // ---- A: router logits (fp64), experts spread over every CTA
    for (int e = warp * G + cta; e < E; e += DF_WARPS * G) {
        double acc[DF_TN], ab[DF_TN];
#pragma unroll
        for (int t = 0; t < DF_TN; ++t) acc[t] = ab[t] = 0.0;
        const float4* w4 = reinterpret_cast<const float4*>(a.W + (size_t)e * H);
#pragma unroll 4
        for (int i = lane; i < H / 4; i += 32) {
            const float4 w = __ldg(w4 + i);
            const double w0 = w.x, w1 = w.y, w2 = w.z, w3 = w.w;
#pragma unroll
            for (int t = 0; t < DF_TN; ++t) {
                if (t < T) {
                    const uint2 xv = __ldg(reinterpret_cast<const uint2*>(a.x + (size_t)t * H) + i);
                    const double x0 = __uint_as_float(xv.x << 16), x1 = __uint_as_float(xv.x & 0xffff0000u);
                    const double x2 = __uint_as_float(xv.y << 16), x3 = __uint_as_float(xv.y & 0xffff0000u);
                    acc[t] = fma(x0, w0, acc[t]);
                    acc[t] = fma(x1, w1, acc[t]);
                    acc[t] = fma(x2, w2, acc[t]);
                    acc[t] = fma(x3, w3, acc[t]);
                    ab[t] += fabs(x0 * w0) + fabs(x1 * w1) + fabs(x2 * w2) + fabs(x3 * w3);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < DF_TN; ++t) {
            acc[t] = warp_sum_d(acc[t]);
            ab[t] = warp_sum_d(ab[t]);
        }
        if (lane == 0) {
            const double bb = a.b ? (double)a.b[e] : 0.0;
            for (int t = 0; t < T; ++t) {
                a.logit[(size_t)t * E + e] = acc[t] + bb;
                a.absum[(size_t)t * E + e] = ab[t] + fabs(bb);
            }
        }
    }
    alive = grid_barrier(a.bar, (unsigned)G, 1);  // uniform across the CTA

    // ---- B: certified top-k of every token (same result in every CTA) and grouping
    if (alive) {
        if (warp < T) {
            TopkArgs ta{};
            ta.x = a.x; ta.W = a.W; ta.b = a.b; ta.logit = a.logit; ta.absum = a.absum;
            ta.gfast = (double)(H / 32 + 6) * 1.1102230246251565e-16 * 1.01;
            ta.T = T; ta.H = H; ta.E = E; ta.k = k;
            int* cs = reinterpret_cast<int*>(ring) + warp * MOE_MAX_E;  // ring is free during B
            double* cvs = reinterpret_cast<double*>(ring + DF_TN * MOE_MAX_E * 4) + warp * MOE_MAX_E;
            topk_token<true>(ta, warp, rt->idx + warp * k, rt->w + warp * k, cs, cvs, cta == 0 ? a.nrechk : nullptr);
        }
        for (int e = tid; e < MOE_MAX_E; e += DF_THREADS) s_cnt[e] = 0;
        __syncthreads();
        for (int p = tid; p < P; p += DF_THREADS) atomicAdd(&s_cnt[rt->idx[p]], 1);
        __syncthreads();
        const int c = tid < E ? s_cnt[tid] : 0;
        int off;
        const int total = block_excl_scan(c, &off, s_warp);
        if (tid < E) s_off[tid] = off;
        int upos;
        const int nu = block_excl_scan((tid < E && c > 0) ? 1 : 0, &upos, s_warp);
        if (tid < E && c > 0) {
            rt->u_e[upos] = tid;
            rt->u_pos[upos] = off;
            rt->u_n[upos] = c;
        }
        if (tid == 0) rt->n_uniq = nu;
        if (cta == 0) {
            if (tid < E) {
                a.offsets[tid] = off;
                if (a.hist) a.hist[(size_t)a.layer * E + tid] += (uint32_t)c;
                if (c > 0) {
                    const int64_t sl = a.slot_table[(int64_t)a.layer * E + tid];
                    if (sl < 0 || sl >= a.n_slots) moe_set_status(MOE_ERR_SLOT);
                }
            }
            if (tid == 0) a.offsets[E] = total;
        }
        __syncthreads();
        for (int p = tid; p < P; p += DF_THREADS) {
            const int e = rt->idx[p];
            int before = 0;
            for (int q2 = 0; q2 < p; ++q2) before += (rt->idx[q2] == e);
            const int pos = s_off[e] + before;
            rt->perm[pos] = p;
            rt->inv[p] = pos;
            if (cta == 0) {
                a.perm[pos] = p;
                a.idx[p] = e;
                a.w[p] = rt->w[p];
            }
        }
        __syncthreads();
    }

    // ---- C: gate/up + SwiGLU over this CTA's range of 16-row tiles
    const int tiles_per_e = I / 16;
    const int nuq = alive ? rt->n_uniq : 0;
    const int R = nuq * tiles_per_e;
    const int r0 = (int)((int64_t)cta * R / G), r1 = (int)((int64_t)(cta + 1) * R / G);
    const int nloc = r1 - r0;
    const int chunk = a.chunk, nch = H / chunk;
    const int nbox_g = chunk * BG / 8 / 128, nbox_u = chunk * BU / 8 / 128;
    const uint32_t bytes_c = (uint32_t)((nbox_g + nbox_u) * 2048 + 2 * 16 * (chunk / 32) * 2);
    const int nunit_c = nloc * nch;
    const int ft0 = cta * DF_FT;  // phase-D features of this CTA
    const bool has_d = alive && ft0 < H;
    const int rowb_d = I * BD / 8;

    if (has_d)  // W_d rows of phase D into L2 while gate/up streams from HBM
        for (int ft = ft0; ft < H; ft += G * DF_FT)
            for (int ui = tid; ui < nuq; ui += DF_THREADS) {
                const int64_t sl = a.slot_table[(int64_t)a.layer * E + rt->u_e[ui]];
                if (sl < 0 || sl >= a.n_slots) continue;
                const uint8_t* base = a.arena + sl * a.slot_bytes;
                prefetch_l2(base + a.off_codes[2] + (int64_t)ft * rowb_d, (uint32_t)(DF_FT * rowb_d));
                prefetch_l2(base + a.off_scales[2] + (int64_t)ft * (I / 32) * 2, (uint32_t)(DF_FT * (I / 32) * 2));
            }

    if (warp == 0) {
        if (lane == 0 && alive) {
            // units go out in rounds of up to 15 tiles (one per consumer warp),
            // chunk-major inside a round, so each warp's units arrive in order
            for (int i = 0; i < nunit_c; ++i) {
                const int s = i % DF_STAGES, ph = (i / DF_STAGES) & 1;
                const int rb = (i / (nch * (DF_WARPS - 1))) * (DF_WARPS - 1);  // first tile of the round
                const int nr = min(DF_WARPS - 1, nloc - rb), w = i - rb * nch;  // unit within the round
                const int gt = r0 + rb + w % nr, ch = w / nr;
                const int ui = gt / tiles_per_e, r16 = gt % tiles_per_e;
                const int64_t sl = a.slot_table[(int64_t)a.layer * E + rt->u_e[ui]];
                if (!mbar_wait(&empty[s], ph ^ 1, 3, i)) { alive = false; break; }
                uint8_t* dst = ring + s * DF_SLOT;
                if (sl < 0 || sl >= a.n_slots) {  // nothing to load: release the consumer
                    mbar_arrive(&full[s]);
                    slot_seq[s] = i;
                    continue;
                }
                mbar_arrive_expect_tx(&full[s], bytes_c);
                slot_seq[s] = i;
                for (int bx = 0; bx < nbox_g; ++bx)
                    tma_load_3d(dst + bx * 2048, &tcg, &full[s], ch * chunk * BG / 8 + bx * 128, r16 * 16, (int)sl);
                for (int bx = 0; bx < nbox_u; ++bx)
                    tma_load_3d(dst + (nbox_g + bx) * 2048, &tcu, &full[s], ch * chunk * BU / 8 + bx * 128, r16 * 16,
                                (int)sl);
                uint8_t* sdst = dst + (nbox_g + nbox_u) * 2048;
                tma_load_3d(sdst, &tsg, &full[s], ch * chunk / 32, r16 * 16, (int)sl);
                tma_load_3d(sdst + 16 * (chunk / 32) * 2, &tsu, &full[s], ch * chunk / 32, r16 * 16, (int)sl);
            }
        }
    } else if (alive) {
        const int g = lane >> 2, q = lane & 3;
        for (int rb = 0; rb < nloc && alive; rb += DF_WARPS - 1) {
            const int nr = min(DF_WARPS - 1, nloc - rb), l = warp - 1;
            if (l >= nr) break;
            const int lt = rb + l;
            const int gt = r0 + lt, ui = gt / tiles_per_e, r16 = gt % tiles_per_e;
            const int e = rt->u_e[ui], pos0 = rt->u_pos[ui], n = rt->u_n[ui];
            const int64_t sl = a.slot_table[(int64_t)a.layer * E + e];
            const bool valid = sl >= 0 && sl < a.n_slots;
            float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
            for (int ch = 0; ch < nch; ++ch) {
                const int i = rb * nch + ch * nr + l;
                const int s = i % DF_STAGES, ph = (i / DF_STAGES) & 1;
                if (!wait_slot(slot_seq, s, i, 7) || !mbar_wait(&full[s], ph, 4, i)) { alive = false; break; }
                if (valid)
                    gateup_chunk<BG, BU>(ring + s * DF_SLOT, chunk, nbox_g, nbox_u, ch * (chunk / 32), xb, xc, accg,
                                         accu);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            // h of this tile's 16 rows for every pair of the expert (token column t)
            for (int jj = 0; jj < n; ++jj) {
                const int pos = pos0 + jj, t = rt->perm[pos] / k;
                const bool mine = (t >> 1) == q;
                const int sel = t & 1;
                float h0 = 0.f, h1 = 0.f;  // rows g, g + 8
                if (mine && valid) {
                    h0 = silu_f32(sel ? accg[1] : accg[0]) * (sel ? accu[1] : accu[0]);
                    h1 = silu_f32(sel ? accg[3] : accg[2]) * (sel ? accu[3] : accu[2]);
                }
                const uint16_t b0 = f32_to_bf16_bits(h0), b1 = f32_to_bf16_bits(h1);
                float part = bf16_bits_to_f32(b0) + bf16_bits_to_f32(b1);
                part += __shfl_xor_sync(0xffffffffu, part, 4);
                part += __shfl_xor_sync(0xffffffffu, part, 8);
                part += __shfl_xor_sync(0xffffffffu, part, 16);
                if (mine) {
                    // element rr of I lands at block rr/32, quad (rr%32)/8, fragment slot of rr%8
                    const int rows[2] = {r16 * 16 + g, r16 * 16 + g + 8};
                    const uint16_t vals[2] = {b0, b1};
#pragma unroll
                    for (int z = 0; z < 2; ++z) {
                        const int rr = rows[z], e32 = rr & 31, i8 = e32 & 7;
                        a.hB[(size_t)pos * I + (rr & ~31) + (e32 >> 3) * 8 + (i8 & 3) * 2 + (i8 >> 2)] = vals[z];
                    }
                    if (g == 0) a.hC[(size_t)pos * (I / 16) + r16] = part;
                }
            }
        }
    }
    {
        const int mine_ok = alive ? 1 : 0;
        const bool gb = grid_barrier(a.bar, 2u * (unsigned)G, 2);
        alive = __syncthreads_and(mine_ok && gb) != 0;
    }

    // ---- D: down projection for this CTA's feature tiles (16 features each), every selected expert; combine
    if (alive) {
        const int nbox_d = rowb_d / 128;
        const uint32_t bytes_d = (uint32_t)(nbox_d * 2048 + 16 * (I / 32) * 2);
        int unit = nunit_c;  // ring units continue from phase C
        for (int ft = ft0; ft < H; ft += G * DF_FT, unit += nuq) {
            if (warp == 0) {
                if (lane == 0) {
                    for (int ui = 0; ui < nuq; ++ui) {
                        const int i = unit + ui;
                        const int s = i % DF_STAGES, ph = (i / DF_STAGES) & 1;
                        const int64_t sl = a.slot_table[(int64_t)a.layer * E + rt->u_e[ui]];
                        if (!mbar_wait(&empty[s], ph ^ 1, 5, i)) break;
                        uint8_t* dst = ring + s * DF_SLOT;
                        if (sl < 0 || sl >= a.n_slots) {
                            mbar_arrive(&full[s]);
                            slot_seq[s] = i;
                            continue;
                        }
                        mbar_arrive_expect_tx(&full[s], bytes_d);
                        slot_seq[s] = i;
                        for (int bx = 0; bx < nbox_d; ++bx)
                            tma_load_3d(dst + bx * 2048, &tcd, &full[s], bx * 128, ft, (int)sl);
                        tma_load_3d(dst + nbox_d * 2048, &tsd, &full[s], 0, ft, (int)sl);
                    }
                }
            } else {
                const int g = lane >> 2, q = lane & 3;
                for (int ui = warp - 1; ui < nuq; ui += DF_WARPS - 1) {
                    const int i = unit + ui;
                    const int s = i % DF_STAGES, ph = (i / DF_STAGES) & 1;
                    const int pos0 = rt->u_pos[ui], n = rt->u_n[ui];
                    const int64_t sl = a.slot_table[(int64_t)a.layer * E + rt->u_e[ui]];
                    const bool valid = sl >= 0 && sl < a.n_slots;
                    if (!wait_slot(slot_seq, s, i, 8) || !mbar_wait(&full[s], ph, 6, i)) break;
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
                    if (valid) down_unit<BD>(a, ring + s * DF_SLOT, nbox_d, pos0, n, acc);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[s]);
                    // y for pair columns 2q, 2q+1 (when they exist), features g, g+8
#pragma unroll
                    for (int z = 0; z < 2; ++z) {
                        const int jj = 2 * q + z;
                        if (jj < n) {
                            const int pos = pos0 + jj;
                            const float wv = rt->w[rt->perm[pos]];
                            ypair[pos * DF_FT + g] = wv * acc[z];
                            ypair[pos * DF_FT + g + 8] = wv * acc[2 + z];
                        }
                    }
                }
            }
            __syncthreads();
            for (int u = tid; u < T * DF_FT; u += DF_THREADS) {
                const int t = u / DF_FT, fl = u % DF_FT, f = ft + fl;
                float sum = 0.f;
                for (int j = 0; j < k; ++j) sum += ypair[rt->inv[t * k + j] * DF_FT + fl];
                if (a.residual) sum = bf16_bits_to_f32(a.x[(size_t)t * H + f]) + sum;
                a.out[(size_t)t * H + f] = f32_to_bf16_bits(sum);
            }
            __syncthreads();
        }
    }
}
