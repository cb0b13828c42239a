// Decode window (T <= 8 tokens) as one persistent, cooperatively launched
// kernel per layer: one CTA per SM, two grid-wide barriers.
//
//   A  router logits in fp64 on the tensor cores (mma.m8n8k4.f64): each CTA
//      takes a few experts; their W_r rows and the window's x arrive by bulk
//      copies into shared memory
//   -- barrier --
//   B  every CTA certifies the top-k of every token (the same deterministic
//      computation everywhere) and builds the grouping (pairs sorted by
//      expert) in shared memory; CTA 0 writes the routing outputs and the
//      histogram
//   C  gate/up + SwiGLU: each CTA owns a contiguous range of 16-row tiles of
//      the selected experts, cut into units of 16 rows x one 128-byte code
//      box per matrix.  Every warp owns a contiguous run of those units and
//      streams them itself through two private TMA slots: it waits for a
//      unit, copies it into registers, re-arms the slot with its next unit
//      and only then computes, so both slots of every warp are in flight
//      almost all the time.  Partial tile sums go to shared memory and are
//      finished (SwiGLU, bf16 h) once the CTA's warps are done.  A warp that
//      runs out of C units already loads its first W_d units.
//   -- barrier --
//   D  down + combine: each CTA owns 16 output features (a feature tile) for
//      every selected expert, so it holds complete sums and writes out[t][f]
//      directly, in a fixed slot order.  h of every pair is copied into
//      shared memory from L2; warps take experts round-robin with the same
//      two-slot streaming.
//
// The dot products run on mma.sync m16n8k16 (bf16 in, fp32 out) with the
// weights as A (16 rows) and the tokens (or an expert's pairs) as the 8
// columns of B, so a weight costs its unpack and one lane-slot of an MMA.
// Codes enter the MMA as (128 + q) in bf16 (an exponent-bias bit pattern:
// 0x4300 | q), so each block's MMA result is sum q x + 128 sum x; the block
// correction (128 + offset) * sum x enters as the MMA's C input and the
// block scale is applied in fp32.  All waits (mbarriers, grid barriers) are
// bounded.
#pragma once
#include "common.cuh"
#include "perm.cuh"
#include "router.cuh"

// Phase timestamps for measurement builds (-DMOE_PROBE): thread 0 of every
// CTA records the global timer at the phase boundaries.  Compiled out
// otherwise.
#ifdef MOE_PROBE
__device__ unsigned long long g_df_probe[160][16];
#define DF_MARK(i)                                                                  \
    do {                                                                            \
        if (threadIdx.x == 0 && blockIdx.x < 160) {                                 \
            unsigned long long t_;                                                  \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                  \
            g_df_probe[blockIdx.x][i] = t_;                                         \
        }                                                                           \
    } while (0)
#else
#define DF_MARK(i) \
    do {           \
    } while (0)
#endif

#define DF_WARPS 16
#define DF_THREADS (32 * DF_WARPS)
#define DF_NBUF 2          // TMA slots per warp
#define DF_CODE_SLOT 4096  // two code boxes of 16 rows x 128 B (128-byte swizzle)
#define DF_TN 8            // token columns of the MMA
#define DF_MAXP 256        // pairs T * k
#define DF_FT 16           // features per phase-D tile
#define DF_MAX_EPC 8       // router experts per CTA (rows of the fp64 MMA)
#define DF_MAX_NBD 16      // quant blocks of a W_d row (I <= 512)
#define DF_SMEM_LIMIT (227 * 1024)
#define DF_BAR_WORDS (32 * 18)  // grid barrier: 16 group counters, the top counter, the flag
#define DF_NREP 8          // copies of the (logit, bound) records that phase B reads

// Shared-memory layout, computed on the host (df_plan) and passed in; offsets
// are from the 1024-byte aligned base of dynamic shared memory.
struct DfPlan {
    int sc_off, sc_slot;        // scale ring [DF_WARPS][DF_NBUF][sc_slot]
    int r1_off;                 // C: xb, xc, partials | D: h, hsum, ypair
    int xc_off, part_off, n_part, part_bytes;
    int hs_stride, hsum_off, ypair_off;
    int route_off, stab_off, bar_off, total;
    // phase A (code ring, free then): x rows, W_r rows, per-warp sums, x block sums
    int a_ws_off, a_sp_off, a_w2_off, a_xp_off;
    // phase B (code ring): per-token scratch, expert counts and offsets
    int b_cnt_off, b_off_off;
};

struct DecodeFusedArgs {
    const uint8_t* arena;
    const int32_t* slot_table;
    int64_t n_slots;
    int64_t off_codes[3], off_scales[3];
    int64_t slot_bytes;
    int H, I, E, k, layer, T, residual;
    int bits_gate, bits_up, bits_down;
    int epc;                 // router experts per CTA
    const uint16_t* x;       // [T][H]
    const float* W;          // router [E][H]
    const float* b;          // router bias [E] or null
    uint16_t* out;           // [T][H]
    float* hout;             // [T][H] fp32 output rows before rounding (steering: a second kernel
                             // finishes them), or null: bf16 rows go straight to out
    uint32_t* hist;          // [L][E] or null
    int32_t* idx;            // [T*k]
    float* w;                // [T*k]
    int32_t* offsets;        // [E+1]
    int32_t* perm;           // [T*k]
    int32_t* nrechk;         // [1]
    double* logit;           // [T][E] workspace
    float* wnorm;            // [E] upper bounds of ||W[e]||_2 (workspace)
    double2* rec;            // [DF_NREP][T][E] (logit, error bound): CTA c reads copy c % DF_NREP
    uint16_t* hB;            // [P][I] bf16, MMA-fragment order within each 32-block
    unsigned int* bar;       // grid barrier counters and flag, DF_BAR_WORDS words (zeroed before launch)
    unsigned spin_limit;     // polling bound of the grid barriers (MOE_SPIN_LIMIT; lowered only by a test)
    unsigned bar1_extra;     // 0; a test sets it to make grid barrier 1 unsatisfiable
    DfPlan pl;
};

__host__ __device__ inline int df_al(int v, int a) { return (v + a - 1) / a * a; }

// Codes per K-chunk of a gate/up unit: one 128-byte box row.
__host__ __device__ constexpr int df_ck(int bits) { return 1024 / bits; }

// Feature tiles of CTA c (tiles c, c + G, ...).
__host__ __device__ inline int df_nft(int c, int NFT, int G) { return c < NFT ? (NFT - 1 - c) / G + 1 : 0; }

// Upper bound of the 16-row gate/up tiles any CTA gets (an equal share).
__host__ inline int df_max_tiles(int P, int E, int I, int G) {
    const int nuq = std::min(P, E);
    return (nuq * (I / 16) + G - 1) / G + 1;
}

// Returns false when the window does not fit one CTA's shared memory.
__host__ inline bool df_plan(DfPlan& p, int T, int P, int E, int H, int I, int bits_gu, int epc, int G,
                             int max_dyn, int* dyn_bytes) {
    const int ck = df_ck(bits_gu), NB = H / 32;
    p = DfPlan{};
    int o = DF_WARPS * DF_NBUF * DF_CODE_SLOT;
    p.sc_slot = df_al(std::max(2 * 16 * (ck / 32) * 2, 16 * (I / 32) * 2), 128);
    p.sc_off = o;
    o += DF_WARPS * DF_NBUF * p.sc_slot;
    p.r1_off = o;
    // phase C
    const int xb = NB * 4 * T * 16;
    p.xc_off = o + xb;
    p.part_off = p.xc_off + NB * 4 * 16;  // C quads [H/32][4]
    p.part_bytes = 2 * 16 * T * 4;
    p.n_part = df_max_tiles(P, E, I, G) + DF_WARPS;
    const int c_end = p.part_off + p.n_part * p.part_bytes;
    // phase D
    p.hs_stride = I * 2 + 16;
    p.hsum_off = o + P * p.hs_stride;
    p.ypair_off = p.hsum_off + P * (I / 32) * 4;
    const int nftr = (H / DF_FT + G - 1) / G;
    const int d_end = p.ypair_off + nftr * P * DF_FT * 4;
    o = df_al(std::max(c_end, d_end), 16);
    p.route_off = o;
    o += df_al((8 * P + 4) * 4, 16);
    p.stab_off = o;  // this layer's row of the slot table
    o += MOE_MAX_E * 4;
    p.bar_off = o;
    o += (DF_WARPS * DF_NBUF + 2) * 8;
    p.total = df_al(o, 128);
    // phase A inside the code ring: x rows [T][2H + 16], W_r rows [epc][4H + 16], sums
    p.a_ws_off = df_al(T * (2 * H + 16), 128);
    p.a_sp_off = df_al(p.a_ws_off + epc * (4 * H + 16), 128);
    p.a_w2_off = p.a_sp_off + DF_WARPS * 64 * 8;
    p.a_xp_off = p.a_w2_off + DF_WARPS * DF_TN * 4;
    // phase B inside the code ring: per-token scratch (6 KB each), counts, offsets
    p.b_cnt_off = DF_TN * MOE_MAX_E * 12;
    p.b_off_off = p.b_cnt_off + MOE_MAX_E * 4;
    *dyn_bytes = 1024 + p.total;
    if (p.a_xp_off + NB * 4 * T * 8 > DF_WARPS * DF_NBUF * DF_CODE_SLOT) return false;
    if (p.b_off_off + MOE_MAX_E * 4 > DF_WARPS * DF_NBUF * DF_CODE_SLOT) return false;
    return *dyn_bytes <= max_dyn;
}

// ---------------------------------------------------------------- small helpers

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier over gridDim.x co-resident CTAs, phase `ph` (1, 2, ...),
// in two levels so that no counter sees more than ~16 arrivals: CTA c arrives
// on group counter c % DF_BAR_GROUPS; the last arrival of a group arrives on
// the top counter; the last arrival there stores the phase to the release
// flag, which the others poll.  Counters and flag sit on separate 128-byte
// lines of `bar` (zeroed before launch) and only grow.  Bounded: on expiry the
// status word gets MOE_ERR_TIMEOUT and every thread of the CTA sees false.
#define DF_BAR_GROUPS 16
// spin_limit bounds the polling (MOE_SPIN_LIMIT unless a test lowers it);
// extra > 0 (a test setting) makes the barrier wait for arrivals that never
// come, so that every waiter runs into that bound.
__device__ __forceinline__ bool grid_barrier(unsigned* bar, unsigned ph, int site, unsigned spin_limit,
                                             unsigned extra = 0) {
    __syncthreads();
    int ok = 1;
    if (threadIdx.x == 0) {
        const unsigned G = gridDim.x, NG = min(G, (unsigned)DF_BAR_GROUPS), grp = blockIdx.x % NG;
        const unsigned members = (G - grp + NG - 1) / NG + extra;
        unsigned* flag = bar + 32 * (DF_BAR_GROUPS + 1);
        __threadfence();
        if (atomicAdd(bar + 32 * grp, 1u) + 1u == ph * members &&
            atomicAdd(bar + 32 * DF_BAR_GROUPS, 1u) + 1u == ph * NG) {
            asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(ph) : "memory");
        } else {
            unsigned it = 0;
            while (ld_acquire_u32(flag) < ph) {
                if (++it > spin_limit) { moe_note_timeout(site, (int)(ld_acquire_u32(flag) % 1000)); ok = 0; break; }
                if (it > 16) __nanosleep(32);
            }
        }
        __threadfence();
    }
    return __syncthreads_and(ok) != 0;
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

// D(4 fp32) += A(16x16 bf16) * B(16x8 bf16).  (Not volatile: a pure function
// of its operands, which the compiler may schedule freely.)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D(4 fp32) = A(16x16 bf16) * B(16x8 bf16) + C, with C a separate register
// quad (loaded as one 16-byte value, so no copies into D are needed).
__device__ __forceinline__ void mma_bf16_16816_c(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                 uint32_t b0, uint32_t b1, const float4& c) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c.x), "f"(c.y), "f"(c.z), "f"(c.w));
}

// Byte offset, inside a 16-row box of 128-byte rows written with the TMA
// 128-byte swizzle, of byte `off` of a row whose swizzle key is
// key16 = (row & 7) << 4: the swizzle XORs the 16-byte chunk index with the
// row's low 3 bits.
__device__ __forceinline__ int sw128(int off, int key16) { return ((off & ~15) ^ key16) | (off & 15); }

// 8 codes of thread q in quant block j of a row: 4 bytes at 4 bits, 2 at 2 bits.
template <int BITS>
__device__ __forceinline__ uint32_t ld_codes(const uint8_t* row, int j, int q, int key16) {
    const int off = j * (32 * BITS / 8) + q * BITS;
    const uint8_t* p = row + (off >> 7) * 2048 + sw128(off & 127, key16);
    if (BITS == 4) return *reinterpret_cast<const uint32_t*>(p);
    return *reinterpret_cast<const uint16_t*>(p);
}

// Four 8x8 b16 matrices from shared memory: lane l gives the address of row
// l % 8 of matrix l / 8 (16 bytes); register k of lane l receives bytes
// 4 (l % 4) .. 4 (l % 4) + 3 of row l / 4 of matrix k.
__device__ __forceinline__ void ldsm_x4(const void* row_addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(row_addr)));
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

// Position of element i (0..I) of a row of h in the fragment order.
__device__ __forceinline__ int frag_pos(int i) {
    const int e32 = i & 31, i8 = e32 & 7;
    return (i & ~31) + (e32 >> 3) * 8 + (i8 & 3) * 2 + (i8 >> 2);
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, uint64_t* bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
            "r"(smem_u32(dst)),
        "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* tm, uint64_t* bar, int c0, int c1, int c2,
                                            int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];" ::
            "r"(smem_u32(dst)),
        "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* tm, uint64_t* bar, int c0, int c1, int c2,
                                            int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::
            "r"(smem_u32(dst)),
        "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
        : "memory");
}

// 16 bytes global -> shared through L2 (cp.async, the LSU path).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// The mbarrier's current phase also waits for this thread's earlier cp.async
// copies (its pending count is raised now and lowered when they land).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

__device__ __forceinline__ float half_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu))); }
__device__ __forceinline__ float half_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }
__device__ __forceinline__ uint32_t u4_word(const uint4& v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

struct DfRoute {  // grouping of the window's pairs, identical in every CTA; arrays of P
    int32_t* idx;    // expert of pair p = t*k + j
    float* w;
    int32_t* perm;   // position -> pair
    int32_t* inv;    // pair -> position
    int32_t* u_e;    // selected experts, ascending
    int32_t* u_pos;  // first position of each
    int32_t* u_n;    // pairs of each
    int32_t* u_sl;   // arena slot of each, -1 when the slot table has none
    int32_t* n_uniq;
};

// ---------------------------------------------------------------- phase B: top-k of one token

// The selection of topk_token<2> with a shorter first step.  Lanes hold
// experts e = lane + 32 i, read as (logit, error bound) records.  Every entry
// at or above theta, the M-th largest of the 32 lane maxima, is a candidate:
// at least M entries (the lane maxima themselves) reach theta, so the
// candidates contain the M largest.  With at most 32 of them they are
// compacted one per lane, sorted by (logit desc, expert asc) and certified as
// in topk_token; otherwise, or when the certification fails, topk_token<2>
// decides from scratch (its exact fallback included).  Loops are unrolled so
// that the shuffles of one step overlap.
__device__ __forceinline__ void df_topk_token(const TopkArgs& a, const double2* rec, int t, int32_t* idx_out,
                                              float* w_out, int* cs, double* cvs, int32_t* nrechk) {
    const int lane = threadIdx.x & 31;
    const int E = a.E, k = a.k;
    constexpr int NV = MOE_MAX_E / 32;
    double v[NV], dl[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        double2 r = make_double2(-INFINITY, 0.0);
        if (e < E) r = __ldcg(rec + e);
        v[i] = order_val(r.x);
        dl[i] = order_bnd(r.y);
    }
    const int M = min(min(E, k + MOE_CAND_EXTRA), 32);
    double m = -INFINITY;
#pragma unroll
    for (int i = 0; i < NV; ++i) m = fmax(m, v[i]);
    int r = 0;  // rank of this lane's maximum (descending, ties by lane)
#pragma unroll 4
    for (int j = 0; j < 32; ++j) {
        const double o = __shfl_sync(0xffffffffu, m, j);
        r += (o > m || (o == m && j < lane)) ? 1 : 0;
    }
    const unsigned sel = __ballot_sync(0xffffffffu, r == M - 1);
    const double th = __shfl_sync(0xffffffffu, m, __ffs(sel) - 1);
    unsigned bm[NV];
    double rest = -INFINITY;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const bool valid = lane + 32 * i < E;
        const bool in = valid && v[i] >= th;
        bm[i] = __ballot_sync(0xffffffffu, in);
        if (valid && !in) rest = fmax(rest, hi_end(v[i], dl[i]));
    }
    int nc = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        if ((bm[i] >> lane) & 1u) {
            const int pos = nc + __popc(bm[i] & ((1u << lane) - 1));
            if (pos < 32) {
                cs[pos] = lane + 32 * i;
                cvs[pos] = v[i];
                cvs[32 + pos] = dl[i];
            }
        }
        nc += __popc(bm[i]);
    }
    rest = warp_max_d(rest);
    __syncwarp();
    if (nc <= 32) {
        double cval = -INFINITY, cbnd = 0.0;
        int ce = 0x7fffffff;
        if (lane < nc) {
            cval = cvs[lane];
            cbnd = cvs[32 + lane];
            ce = cs[lane];
        }
        // position of this candidate in (value desc, expert asc) order
        int rank = 0;
#pragma unroll 4
        for (int j = 0; j < 32; ++j) {
            const double oj = __shfl_sync(0xffffffffu, cval, j);
            const int ej = __shfl_sync(0xffffffffu, ce, j);
            rank += (j < nc && (oj > cval || (oj == cval && ej < ce))) ? 1 : 0;
        }
        __syncwarp();
        if (lane < nc) {  // scatter into sorted order through the scratch
            cvs[rank] = cval;
            cvs[32 + rank] = cbnd;
            cs[rank] = ce;
        }
        __syncwarp();
        if (lane < nc) {
            cval = cvs[lane];
            cbnd = cvs[32 + lane];
            ce = cs[lane];
        }
        const double nv = __shfl_down_sync(0xffffffffu, cval, 1);
        const double nb = __shfl_down_sync(0xffffffffu, cbnd, 1);
        bool ok = true;
        if (lane < k && lane + 1 < nc) ok = lo_end(cval, cbnd) > hi_end(nv, nb);
        if (lane == k - 1) ok = ok && (rest == -INFINITY || lo_end(cval, cbnd) > rest);
        if (__all_sync(0xffffffffu, ok)) {
            write_topk(k, cval, ce, idx_out, w_out);
            return;
        }
    }
    __syncwarp();
    topk_token<2>(a, t, idx_out, w_out, cs, cvs, nrechk);
}

// ---------------------------------------------------------------- L2 prefetch of a selected expert

// This CTA's 1/G slice [lo, lo + n) of expert slot `sl`, prefetched into L2.
// Every CTA issues its slice of each selected expert as soon as a token's
// selection is known, so the window's expert bytes start streaming from HBM
// before the grouping is built and the first unit is requested; the units'
// own loads then find them in L2 (or already in flight).
__device__ __forceinline__ void df_prefetch_slot(const DecodeFusedArgs& a, int sl, uint32_t lo, uint32_t n) {
    if (n > 0) prefetch_l2(a.arena + (int64_t)sl * a.slot_bytes + lo, n);
}

// ---------------------------------------------------------------- phase C: one gate/up unit

// A unit is 16 rows x CK = 1024 / BITS codes of W_g and of W_u (one 128-byte
// box row each) and their scales.  Lane (g, q) keeps the codes it feeds to the
// MMA (rows g and g + 8; at 2 bits two blocks share a word) and its scales.
template <int BITS>
struct DfCRegs {
    static constexpr int NB = 32 / BITS;  // quant blocks per unit
    uint32_t g0[8], g1[8], u0[8], u1[8];
    uint4 sg0[NB / 8], sg1[NB / 8], su0[NB / 8], su1[NB / 8];
};

template <int BITS>
__device__ __forceinline__ void df_stage_c(const uint8_t* code, const uint8_t* sc, DfCRegs<BITS>& r) {
    constexpr int NB = DfCRegs<BITS>::NB, NS = NB / 8;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3, key16 = (g & 7) << 4;
    if (BITS == 4) {
        // block j of gate rows 0-7 / 8-15, up rows 0-7 / 8-15: one 16-byte chunk per row
        const int rr = lane & 7;
        const uint8_t* rowp = code + (lane >> 4) * 2048 + ((lane >> 3) & 1) * 1024 + rr * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) ldsm_x4(rowp + ((j ^ rr) << 4), r.g0[j], r.g1[j], r.u0[j], r.u1[j]);
    } else {
        const uint8_t* rg0 = code + g * 128;
        const uint8_t* ru0 = code + 2048 + g * 128;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            r.g0[w] = ld_codes<2>(rg0, 2 * w, q, key16) | (ld_codes<2>(rg0, 2 * w + 1, q, key16) << 16);
            r.g1[w] = ld_codes<2>(rg0 + 1024, 2 * w, q, key16) | (ld_codes<2>(rg0 + 1024, 2 * w + 1, q, key16) << 16);
            r.u0[w] = ld_codes<2>(ru0, 2 * w, q, key16) | (ld_codes<2>(ru0, 2 * w + 1, q, key16) << 16);
            r.u1[w] = ld_codes<2>(ru0 + 1024, 2 * w, q, key16) | (ld_codes<2>(ru0 + 1024, 2 * w + 1, q, key16) << 16);
        }
    }
    const uint4* sg = reinterpret_cast<const uint4*>(sc);  // [16 rows][NB] fp16, gate then up
    const uint4* su = sg + 16 * NS;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        r.sg0[i] = sg[g * NS + i];
        r.sg1[i] = sg[(g + 8) * NS + i];
        r.su0[i] = su[g * NS + i];
        r.su1[i] = su[(g + 8) * NS + i];
    }
}

__device__ __forceinline__ float df_scale(const uint4* s, int j) {
    const uint32_t w = u4_word(s[j >> 3], (j & 7) >> 1);
    return (j & 1) ? half_hi(w) : half_lo(w);
}

// accg / accu (rows g, g + 8; token columns 2q, 2q + 1) += the unit's blocks
// J0 .. J0 + NB - 1.  xb: x fragments [H/32][4][T]; xc: per (block, lane q)
// the MMA's C quad (c_2q, c_2q+1, c_2q, c_2q+1), c = -(128 + offset) sum x.
template <int BITS>
__device__ __forceinline__ void df_compute_c(const DfCRegs<BITS>& r, const uint4* xb, const float4* xc, int J0, int T,
                                             float (&accg)[4], float (&accu)[4]) {
    constexpr int NB = DfCRegs<BITS>::NB;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
        const int J = J0 + j;
        uint4 bx = make_uint4(0u, 0u, 0u, 0u);
        if (g < T) bx = xb[(J * 4 + q) * T + g];
        const float4 c = xc[J * 4 + q];
        const int sh = BITS == 2 ? 16 * (j & 1) : 0;
        const int wi = BITS == 2 ? (j >> 1) : j;
        uint32_t pg0[4], pg1[4], pu0[4], pu1[4];
        unpack8<BITS>(r.g0[wi] >> sh, pg0);
        unpack8<BITS>(r.g1[wi] >> sh, pg1);
        unpack8<BITS>(r.u0[wi] >> sh, pu0);
        unpack8<BITS>(r.u1[wi] >> sh, pu1);
        float dg[4], du[4];
        mma_bf16_16816_c(dg, pg0[0], pg1[0], pg0[1], pg1[1], bx.x, bx.y, c);
        mma_bf16_16816_c(du, pu0[0], pu1[0], pu0[1], pu1[1], bx.x, bx.y, c);
        mma_bf16_16816(dg, pg0[2], pg1[2], pg0[3], pg1[3], bx.z, bx.w);
        mma_bf16_16816(du, pu0[2], pu1[2], pu0[3], pu1[3], bx.z, bx.w);
        const float sg0 = df_scale(r.sg0, j), sg1 = df_scale(r.sg1, j);
        const float su0 = df_scale(r.su0, j), su1 = df_scale(r.su1, j);
        accg[0] = fmaf(sg0, dg[0], accg[0]);
        accg[1] = fmaf(sg0, dg[1], accg[1]);
        accg[2] = fmaf(sg1, dg[2], accg[2]);
        accg[3] = fmaf(sg1, dg[3], accg[3]);
        accu[0] = fmaf(su0, du[0], accu[0]);
        accu[1] = fmaf(su0, du[1], accu[1]);
        accu[2] = fmaf(su1, du[2], accu[2]);
        accu[3] = fmaf(su1, du[3], accu[3]);
    }
}

// ---------------------------------------------------------------- phase D: one expert, one feature tile

// acc (features g, g + 8; pair columns 2q, 2q + 1) = W_d rows ft .. ft + 15 x h
// of the expert's n pairs, straight from the slot in a rolled loop (two
// blocks per step): a W_d unit is used once per launch, so its code stays
// small instead of being unrolled over all blocks.  The unit's codes sit as
// [16 rows][nbox 128-byte chunks] with the TMA 128-byte swizzle keyed on the
// 128-byte line index (row * nbox + chunk); scales as [16 rows][nblk] fp16;
// hs: h of the first pair [n][hstride bytes] in fragment order; hsum: per pair
// and block, the sum of its 32 h values.
template <int BD, int nblk>
__device__ __forceinline__ void df_compute_d_smem(const uint8_t* code, const uint8_t* sc, const uint8_t* hs, int hstride,
                                                  const float* hsum, int n, float (&acc)[4]) {
    constexpr int nbox = nblk * BD / 32;
    constexpr float kOff = 128.f + (float)(1 << (BD - 1));
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3, key16 = (g & 7) << 4;
    const bool col_ok = g < n, ok0 = 2 * q < n, ok1 = 2 * q + 1 < n;
    const int mrow = ((lane >> 3) & 1) * 8 + (lane & 7), jo = lane >> 4;  // ldmatrix row address of this lane
    const uint8_t* hrow = hs + g * hstride + q * 16;
#pragma unroll 1
    for (int j = 0; j < nblk; j += 2) {
        uint32_t c[2][2];  // [block j, j + 1][row g, g + 8]
        if (BD == 4) {
            const int jj = j + jo, line = mrow * nbox + (jj >> 3);
            ldsm_x4(code + line * 128 + (((jj & 7) ^ (line & 7)) << 4), c[0][0], c[0][1], c[1][0], c[1][1]);
        } else {
#pragma unroll
            for (int z = 0; z < 2; ++z) {
                c[z][0] = ld_codes<BD>(code + g * 128, j + z, q, key16);
                c[z][1] = ld_codes<BD>(code + g * 128 + 1024, j + z, q, key16);
            }
        }
        const uint32_t sw0 = *reinterpret_cast<const uint32_t*>(sc + (g * nblk + j) * 2);  // rows g, g + 8
        const uint32_t sw1 = *reinterpret_cast<const uint32_t*>(sc + ((g + 8) * nblk + j) * 2);
#pragma unroll
        for (int z = 0; z < 2; ++z) {
            const int jb = j + z;
            uint4 bx = make_uint4(0u, 0u, 0u, 0u);
            if (col_ok) bx = *reinterpret_cast<const uint4*>(hrow + jb * 64);
            const float h0 = ok0 ? hsum[(2 * q) * nblk + jb] : 0.f;
            const float h1 = ok1 ? hsum[(2 * q + 1) * nblk + jb] : 0.f;
            uint32_t p0[4], p1[4];
            unpack8<BD>(c[z][0], p0);
            unpack8<BD>(c[z][1], p1);
            float d[4] = {-kOff * h0, -kOff * h1, -kOff * h0, -kOff * h1};
            mma_bf16_16816(d, p0[0], p1[0], p0[1], p1[1], bx.x, bx.y);
            mma_bf16_16816(d, p0[2], p1[2], p0[3], p1[3], bx.z, bx.w);
            const float s0 = z ? half_hi(sw0) : half_lo(sw0), s1 = z ? half_hi(sw1) : half_lo(sw1);
            acc[0] = fmaf(s0, d[0], acc[0]);
            acc[1] = fmaf(s0, d[1], acc[1]);
            acc[2] = fmaf(s1, d[2], acc[2]);
            acc[3] = fmaf(s1, d[3], acc[3]);
        }
    }
}

// ---------------------------------------------------------------- the kernel

template <int BGU, int BD, int NBD>
__global__ void __launch_bounds__(DF_THREADS, 1)
    k_decode_fused(const __grid_constant__ CUtensorMap tgu, const __grid_constant__ CUtensorMap tcd,
                   DecodeFusedArgs a) {
    extern __shared__ uint8_t smem_raw[];
    constexpr int CK = df_ck(BGU), NBU = CK / 32;  // codes and quant blocks per gate/up unit
    // 1024-byte aligned base, derived by pointer arithmetic so that every access
    // through it compiles to a shared-memory (not generic) load or store
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const DfPlan& pl = a.pl;
    const int H = a.H, I = a.I, E = a.E, k = a.k, T = a.T, P = T * k, NB = H / 32;
    uint8_t* ring = base;               // code slots [warp][DF_NBUF][DF_CODE_SLOT]
    uint8_t* scr = base + pl.sc_off;    // scale slots [warp][DF_NBUF][sc_slot]
    uint4* xb = reinterpret_cast<uint4*>(base + pl.r1_off);
    float4* xc = reinterpret_cast<float4*>(base + pl.xc_off);
    float* part = reinterpret_cast<float*>(base + pl.part_off);
    DfRoute rt;
    rt.idx = reinterpret_cast<int32_t*>(base + pl.route_off);
    rt.w = reinterpret_cast<float*>(rt.idx + P);
    rt.perm = reinterpret_cast<int32_t*>(rt.w + P);
    rt.inv = rt.perm + P;
    rt.u_e = rt.inv + P;
    rt.u_pos = rt.u_e + P;
    rt.u_n = rt.u_pos + P;
    rt.u_sl = rt.u_n + P;
    rt.n_uniq = rt.u_sl + P;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + pl.bar_off);  // [DF_WARPS][DF_NBUF]
    uint64_t* abar = full + DF_WARPS * DF_NBUF;  // x rows and the slot-table row
    uint64_t* wbar = abar + 1;                   // this CTA's W_r rows
    const int32_t* stab = reinterpret_cast<const int32_t*>(base + pl.stab_off);
    __shared__ int s_warp[33];
    __shared__ float s_xnorm[DF_TN];
    __shared__ float s_wn[DF_MAX_EPC];
    __shared__ int s_ustart[DF_WARPS + 1];  // first gate/up unit of each warp

    const int G = gridDim.x, cta = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < DF_WARPS * DF_NBUF; ++i) mbar_init(&full[i], 1);
        mbar_init(abar, 1);
        mbar_init(wbar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    DF_MARK(0);

    // ---- A: router logits in fp64 on the tensor cores.  This CTA takes experts
    // e0 .. e0 + epc - 1 (rows of mma.m8n8k4.f64); its warps split H.  Every
    // bf16 x fp32 product is exact in fp64, so only the additions round
    // (bound: gamma_(H+32)).  The x rows and the W_r rows come in by bulk copies.
    const int epc = a.epc, e0 = cta * epc;
    const int ne = e0 < E ? min(epc, E - e0) : 0;
    const int xstride = 2 * H + 16, wstride = 4 * H + 16;  // padded rows: conflict-free fragment loads
    uint8_t* xs = ring;
    uint8_t* ws = ring + pl.a_ws_off;
    if (tid == 0) {
        // the arrival completes the phase at once when ne == 0 (no bytes expected)
        mbar_arrive_expect_tx(wbar, (uint32_t)(ne * 4 * H));
        for (int e = 0; e < ne; ++e) bulk_load(ws + e * wstride, a.W + (size_t)(e0 + e) * H, (uint32_t)(4 * H), wbar);
        mbar_arrive_expect_tx(abar, (uint32_t)(T * 2 * H + E * 4));
        for (int t = 0; t < T; ++t) bulk_load(xs + t * xstride, a.x + (size_t)t * H, (uint32_t)(2 * H), abar);
        bulk_load(base + pl.stab_off, a.slot_table + (size_t)a.layer * E, (uint32_t)(E * 4), abar);
    }
    bool alive = mbar_wait(abar, 0, 1, 0);  // the x fragments are built while W_r is still arriving
    DF_MARK(1);
    // x as MMA B fragments [H/32][4][T], its block sums and squares
    float* xp = reinterpret_cast<float*>(ring + pl.a_xp_off);  // [2][H/32][4][T]
    const int nxf = NB * 4 * T;
    for (int u = tid; u < nxf; u += DF_THREADS) {
        const int n = u % T, q = (u / T) % 4, j = u / (4 * T);
        const uint4 r4 = *reinterpret_cast<const uint4*>(xs + n * xstride + (32 * j + 8 * q) * 2);
        float v[8];
        v[0] = __uint_as_float(r4.x << 16); v[1] = __uint_as_float(r4.x & 0xffff0000u);
        v[2] = __uint_as_float(r4.y << 16); v[3] = __uint_as_float(r4.y & 0xffff0000u);
        v[4] = __uint_as_float(r4.z << 16); v[5] = __uint_as_float(r4.z & 0xffff0000u);
        v[6] = __uint_as_float(r4.w << 16); v[7] = __uint_as_float(r4.w & 0xffff0000u);
        xb[u] = frag_order8(v);
        xp[u] = ((((((v[0] + v[1]) + v[2]) + v[3]) + v[4]) + v[5]) + v[6]) + v[7];
        float sq = 0.f;
#pragma unroll
        for (int z = 0; z < 8; ++z) sq = fmaf(v[z], v[z], sq);
        xp[nxf + u] = sq;
    }
    alive = mbar_wait(wbar, 0, 1, 1) && alive;
    DF_MARK(2);
    if (ne > 0) {
        const int g = lane >> 2, q = lane & 3;
        const int kw = H / DF_WARPS, kb = warp * kw;
        const bool erow = g < ne, xrow_ok = g < T;
        const uint8_t* wrow = ws + (erow ? g : 0) * wstride;
        const uint8_t* xrow = xs + (xrow_ok ? g : 0) * xstride;
        double c0 = 0.0, c1 = 0.0;
        float w2 = 0.f;
#pragma unroll 4
        for (int k0 = kb; k0 < kb + kw; k0 += 16) {
            // step s of this 16-element slice uses k = k0 + 4 q + s (A and B alike)
            const float4 wv = erow ? *reinterpret_cast<const float4*>(wrow + (k0 + 4 * q) * 4) : make_float4(0, 0, 0, 0);
            const uint2 xv = xrow_ok ? *reinterpret_cast<const uint2*>(xrow + (k0 + 4 * q) * 2) : make_uint2(0, 0);
            w2 = fmaf(wv.x, wv.x, fmaf(wv.y, wv.y, fmaf(wv.z, wv.z, fmaf(wv.w, wv.w, w2))));
            const double av[4] = {wv.x, wv.y, wv.z, wv.w};
            const double bv[4] = {__uint_as_float(xv.x << 16), __uint_as_float(xv.x & 0xffff0000u),
                                  __uint_as_float(xv.y << 16), __uint_as_float(xv.y & 0xffff0000u)};
#pragma unroll
            for (int st = 0; st < 4; ++st)
                asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                             : "+d"(c0), "+d"(c1)
                             : "d"(av[st]), "d"(bv[st]));
        }
        // c0, c1: expert e0 + g, tokens 2q, 2q+1 (this warp's slice of H)
        double* sp = reinterpret_cast<double*>(ring + pl.a_sp_off);
        sp[(warp * 8 + g) * 8 + 2 * q] = c0;
        sp[(warp * 8 + g) * 8 + 2 * q + 1] = c1;
        w2 += __shfl_xor_sync(0xffffffffu, w2, 1);
        w2 += __shfl_xor_sync(0xffffffffu, w2, 2);
        float* sw2 = reinterpret_cast<float*>(ring + pl.a_w2_off);
        if (q == 0) sw2[warp * 8 + g] = w2;
    }
    __syncthreads();
    if (warp < T) {  // ||x_t|| for the top-k bounds (inflated over its fp32 rounding)
        float sq = 0.f;
        for (int u = lane; u < NB * 4; u += 32) sq += xp[nxf + u * T + warp];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) s_xnorm[warp] = sqrtf(sq) * 1.001f;
    } else if (warp == T && lane < ne) {  // ||W_r[e]|| of this CTA's experts
        const float* sw2 = reinterpret_cast<const float*>(ring + pl.a_w2_off);
        float s2 = 0.f;
        for (int w = 0; w < DF_WARPS; ++w) s2 += sw2[w * 8 + lane];
        s_wn[lane] = sqrtf(s2) * 1.001f;
        a.wnorm[e0 + lane] = s_wn[lane];
    }
    for (int u = tid; u < NB * 4; u += DF_THREADS) {  // block corrections as MMA C quads, zero beyond T
        const int q = u % 4, j = u / 4;
        float sx[2];
#pragma unroll
        for (int z = 0; z < 2; ++z) {
            const int n = 2 * q + z;
            sx[z] = 0.f;
            if (n < T) {
                const float* pp = xp + (size_t)j * 4 * T + n;
                sx[z] = ((pp[0] + pp[T]) + pp[2 * T]) + pp[3 * T];
            }
        }
        const float f = -(128.f + (float)(1 << (BGU - 1)));
        xc[u] = make_float4(f * sx[0], f * sx[1], f * sx[0], f * sx[1]);
    }
    __syncthreads();
    if (tid < 64 && (tid >> 3) < ne && (tid & 7) < T) {  // logits and their error bounds
        const double* sp = reinterpret_cast<const double*>(ring + pl.a_sp_off);
        const int gg = tid >> 3, t = tid & 7, e = e0 + gg;
        double sum = 0.0;
        for (int w = 0; w < DF_WARPS; ++w) sum += sp[(w * 8 + gg) * 8 + t];
        const double bb = a.b ? (double)a.b[e] : 0.0;
        const double lg = sum + bb;
        a.logit[(size_t)t * E + e] = lg;
        // every sum along a product's path: at most H + 32 roundings in these
        // sums, H + 2 in the definition's own sequential sum
        const double gam = ((double)(H + 32) + (double)(H + 2)) * 1.1102230246251565e-16 * 1.01;
        const double B = ((double)s_xnorm[t] * (double)s_wn[gg] + fabs(bb)) * 1.001;
        const double2 r = make_double2(lg, B * gam + 1e-300);
#pragma unroll
        for (int c = 0; c < DF_NREP; ++c) a.rec[((size_t)c * T + t) * E + e] = r;
    }
    DF_MARK(3);
    {
        const bool gb = grid_barrier(a.bar, 1u, 1, a.spin_limit, a.bar1_extra);
        alive = __syncthreads_and(alive && gb) != 0;  // uniform across the CTA
    }
    DF_MARK(4);

    // ---- B: certified top-k of every token (same result in every CTA) and grouping
    const uint32_t pf_step = (uint32_t)((a.slot_bytes / G + 15) & ~(int64_t)15);
    const uint32_t pf_lo = pf_step * (uint32_t)cta;
    const uint32_t pf_n = pf_lo >= a.slot_bytes ? 0u : (uint32_t)min((int64_t)pf_step, a.slot_bytes - pf_lo);
    if (alive) {
        if (warp < T) {
            TopkArgs ta{};
            ta.x = a.x; ta.W = a.W; ta.b = a.b; ta.logit = a.logit; ta.wnorm = a.wnorm; ta.xnorm = s_xnorm;
            // phase-A sums: at most H + 32 roundings along any product's path
            ta.gfast = (double)(H + 32) * 1.1102230246251565e-16 * 1.01;
            ta.T = T; ta.H = H; ta.E = E; ta.k = k;
            int* cs = reinterpret_cast<int*>(ring + warp * MOE_MAX_E * 12);  // the ring is free during B
            double* cvs = reinterpret_cast<double*>(ring + warp * MOE_MAX_E * 12 + MOE_MAX_E * 4);
            const double2* rec = a.rec + ((size_t)(cta % DF_NREP) * T + warp) * E;
            df_topk_token(ta, rec, warp, rt.idx + warp * k, rt.w + warp * k, cs, cvs, cta == 0 ? a.nrechk : nullptr);
            __syncwarp();
            if (lane < k) {  // this token's experts start streaming into L2
                const int e = rt.idx[warp * k + lane];
                const int64_t sl = (unsigned)e < (unsigned)E ? stab[e] : -1;
                if (sl >= 0 && sl < a.n_slots) df_prefetch_slot(a, (int)sl, pf_lo, pf_n);
            }
        }
        int* s_cnt = reinterpret_cast<int*>(ring + pl.b_cnt_off);
        int* s_off = reinterpret_cast<int*>(ring + pl.b_off_off);
        for (int e = tid; e < MOE_MAX_E; e += DF_THREADS) s_cnt[e] = 0;
        __syncthreads();
        DF_MARK(5);
        for (int p = tid; p < P; p += DF_THREADS) {
            int e = rt.idx[p];
            if ((unsigned)e >= (unsigned)E) {  // never produced by the top-k; a guard against a library fault
                e = 0;
                rt.idx[p] = 0;
                moe_set_status(MOE_ERR_RANGE);
            }
            atomicAdd(&s_cnt[e], 1);
        }
        __syncthreads();
        const int c = tid < E ? s_cnt[tid] : 0;
        int off;
        const int total = block_excl_scan(c, &off, s_warp);
        if (tid < E) s_off[tid] = off;
        int upos;
        const int nu = block_excl_scan((tid < E && c > 0) ? 1 : 0, &upos, s_warp);
        if (tid < E && c > 0) {
            const int64_t sl = stab[tid];
            rt.u_e[upos] = tid;
            rt.u_pos[upos] = off;
            rt.u_n[upos] = c;
            rt.u_sl[upos] = (sl >= 0 && sl < a.n_slots) ? (int32_t)sl : -1;
            if (cta == 0 && rt.u_sl[upos] < 0) moe_set_status(MOE_ERR_SLOT);
        }
        if (tid == 0) *rt.n_uniq = nu;
        if (cta == 0) {
            if (tid < E) {
                a.offsets[tid] = off;
                if (a.hist) a.hist[(size_t)a.layer * E + tid] += (uint32_t)c;
            }
            if (tid == 0) a.offsets[E] = total;
        }
        __syncthreads();
        for (int p = tid; p < P; p += DF_THREADS) {
            const int e = rt.idx[p];
            int before = 0;
            for (int q2 = 0; q2 < p; ++q2) before += (rt.idx[q2] == e);
            const int pos = s_off[e] + before;
            rt.perm[pos] = p;
            rt.inv[p] = pos;
            if (cta == 0) {
                a.perm[pos] = p;
                a.idx[p] = e;
                a.w[p] = rt.w[p];
            }
        }
        __syncthreads();
    }
    DF_MARK(6);

    // ---- C: gate/up + SwiGLU.  A grid barrier separates C from D, so each phase
    // is balanced on its own: every CTA takes an equal share of the 16-row
    // gate/up tiles, contiguous in (expert, row) order.
    const int tiles_e = I / 16, NCH = H / CK, NFT = H / DF_FT;
    constexpr int nblk_d = NBD, nbox_d = NBD * BD / 32;  // W_d row: quant blocks, 128-byte chunks
    const int nuq = alive ? *rt.n_uniq : 0;
    const int R = nuq * tiles_e;
    const int r0 = (int)((int64_t)cta * R / G), r1 = (int)((int64_t)(cta + 1) * R / G);
    const int nloc = r1 - r0;
    if (nloc + DF_WARPS > pl.n_part) {  // the host's bound on partial slots was wrong
        moe_set_status(MOE_ERR_RANGE);
        alive = false;
    }
    // this warp's units: gate/up units [ub, ue) of the CTA's tiles (tile-major),
    // then W_d units (feature round rr, expert warp + 16 i)
    const int Uc = alive ? nloc * NCH : 0;
    if (tid <= DF_WARPS) s_ustart[tid] = tid * Uc / DF_WARPS;
    const int ub = warp * Uc / DF_WARPS, ue = (warp + 1) * Uc / DF_WARPS;
    const int nC = ue - ub;
    const int nftc = df_nft(cta, NFT, G);
    const int ndw = (alive && nuq > warp) ? (nuq - warp + DF_WARPS - 1) / DF_WARPS : 0;
    const int S = nC + nftc * ndw;
    const uint32_t bytes_c = 2u * 2048u, bytes_d = (uint32_t)(nbox_d * 2048);
    const int64_t srow_g = H / 32 * 2, srow_d = nblk_d * 2;  // bytes of a scale row (gate/up, down)

    // Issue unit s of this warp into its slot s % DF_NBUF (all lanes): every
    // lane copies 16 bytes of scales with cp.async, then lane 0 starts one TMA
    // load of the codes.  The slot's barrier completes when both have landed.
    auto issue = [&](int s) {
        const int b = s % DF_NBUF;
        uint64_t* fb = &full[warp * DF_NBUF + b];
        uint8_t* cdst = ring + (warp * DF_NBUF + b) * DF_CODE_SLOT;
        uint8_t* sdst = scr + (warp * DF_NBUF + b) * pl.sc_slot;
        if (s < nC) {
            const int u = ub + s, lt = u / NCH, ch = u % NCH, gt = r0 + lt, ui = gt / tiles_e, r16 = gt % tiles_e;
            const int sl = rt.u_sl[ui];
            if (sl >= 0) {
                // scales [gate, up][16 rows][NBU]: lane l takes row l % 16 of matrix l / 16
                const uint8_t* src = a.arena + (int64_t)sl * a.slot_bytes + a.off_scales[lane >> 4] +
                                     (int64_t)(r16 * 16 + (lane & 15)) * srow_g + ch * NBU * 2;
                uint8_t* dst = sdst + (lane >> 4) * 16 * NBU * 2 + (lane & 15) * NBU * 2;
#pragma unroll
                for (int z = 0; z < NBU / 8; ++z) cp_async16(dst + 16 * z, src + 16 * z);
                cp_async_mbar_arrive(fb);
            }
            __syncwarp();
            if (lane == 0) {
                if (sl < 0) {
                    mbar_arrive(fb);  // nothing to load: the unit counts 0
                } else {
                    mbar_arrive_expect_tx(fb, bytes_c);
                    tma_load_5d(cdst, &tgu, fb, 0, ch, r16 * 16, 0, sl);  // gate and up, 16 rows x 128 B each
                }
            }
        } else {
            const int d = s - nC, rr = d / ndw, ui = warp + DF_WARPS * (d % ndw);
            const int ft = (cta + rr * G) * DF_FT;
            const int sl = rt.u_sl[ui];
            if (sl >= 0) {  // scales [16 rows][nblk_d]: lane l takes 16 bytes of row l % 16
                const int per = (int)(srow_d / 16);  // 16-byte pieces per row (1 or 2)
                if (lane < 16 * per) {
                    const uint8_t* src = a.arena + (int64_t)sl * a.slot_bytes + a.off_scales[2] +
                                         (int64_t)(ft + lane % 16) * srow_d + (lane / 16) * 16;
                    cp_async16(sdst + (lane % 16) * srow_d + (lane / 16) * 16, src);
                }
                cp_async_mbar_arrive(fb);
            }
            __syncwarp();
            if (lane == 0) {
                if (sl < 0) {
                    mbar_arrive(fb);
                } else {
                    mbar_arrive_expect_tx(fb, bytes_d);
                    tma_load_4d(cdst, &tcd, fb, 0, 0, ft, sl);  // 16 rows x nbox_d x 128 B
                }
            }
        }
    };

    int issued = 0;  // units issued by this warp (the same count in every lane)
    if (S > 0) {
        if (lane == 0) fence_proxy_async_smem();  // the ring held generic-proxy data during A and B
        __syncwarp();
        for (; issued < min(S, DF_NBUF); ++issued) issue(issued);
    }
    bool wok = true;
    int s = 0;  // units consumed
    {
        float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
        const int g = lane >> 2, q = lane & 3;
        for (; s < nC; ++s) {
            const int b = s % DF_NBUF;
            if (!mbar_wait(&full[warp * DF_NBUF + b], (uint32_t)(s / DF_NBUF) & 1u, 4, s)) { wok = false; break; }
            if (s == 0) DF_MARK(7);
            const int u = ub + s, lt = u / NCH, ch = u % NCH, gt = r0 + lt, ui = gt / tiles_e;
            const bool valid = rt.u_sl[ui] >= 0;
            DfCRegs<BGU> cr;
            if (valid)
                df_stage_c<BGU>(ring + (warp * DF_NBUF + b) * DF_CODE_SLOT, scr + (warp * DF_NBUF + b) * pl.sc_slot,
                                cr);
            __syncwarp();  // every lane's reads of the slot are done: it may be refilled
            if (issued < S) issue(issued++);  // re-arm the slot with unit s + DF_NBUF
            if (valid) df_compute_c<BGU>(cr, xb, xc, ch * NBU, T, accg, accu);
            if (s == nC - 1 || (u + 1) / NCH != lt) {  // this warp's part of tile lt is complete
                float* pp = part + (size_t)(lt + warp) * (2 * 16 * T);  // [gate, up][16 rows][T]
#pragma unroll
                for (int z = 0; z < 2; ++z) {
                    const int col = 2 * q + z;
                    if (col < T) {
                        pp[g * T + col] = accg[z];
                        pp[(g + 8) * T + col] = accg[2 + z];
                        pp[16 * T + g * T + col] = accu[z];
                        pp[16 * T + (g + 8) * T + col] = accu[2 + z];
                    }
                }
#pragma unroll
                for (int z = 0; z < 4; ++z) accg[z] = accu[z] = 0.f;
            }
        }
    }
    const bool cok = __syncthreads_and(wok && alive) != 0;
    DF_MARK(8);
    // finish the tiles: sum the partials of the warps that covered each tile (in
    // warp order), SwiGLU, round h to bf16 and store it for every pair of the expert
    if (cok) {
        for (int item = tid; item < nloc * 16 * DF_TN; item += DF_THREADS) {
            const int lt = item / (16 * DF_TN), row = (item / DF_TN) % 16, jj = item % DF_TN;
            const int gt = r0 + lt, ui = gt / tiles_e, r16 = gt % tiles_e;
            if (jj >= rt.u_n[ui]) continue;
            const int pos = rt.u_pos[ui] + jj, t = rt.perm[pos] / k;
            const int u_first = lt * NCH, u_end = u_first + NCH;
            float gs = 0.f, us = 0.f;
            for (int w = 0; w < DF_WARPS; ++w) {  // warps whose units meet the tile, in order
                const int wb = s_ustart[w], we = s_ustart[w + 1];
                if (wb >= we || we <= u_first || wb >= u_end) continue;
                const float* pp = part + (size_t)(lt + w) * (2 * 16 * T);
                gs += pp[row * T + t];
                us += pp[16 * T + row * T + t];
            }
            const float h = silu_f32(gs) * us;
            a.hB[(size_t)pos * I + frag_pos(r16 * 16 + row)] = f32_to_bf16_bits(h);
        }
    }
    DF_MARK(9);
    {
        const bool gb = grid_barrier(a.bar, 2u, 2, a.spin_limit);
        alive = __syncthreads_and(cok && gb) != 0;
    }
    DF_MARK(10);

    // ---- D: down projection of this CTA's feature tiles for every selected
    // expert (warp w takes experts w, w + 16, ...), then the combine.
    uint8_t* hs = base + pl.r1_off;  // h of every pair [P][hs_stride], fragment order
    float* hsum = reinterpret_cast<float*>(base + pl.hsum_off);    // [P][I/32]
    float* ypair = reinterpret_cast<float*>(base + pl.ypair_off);  // [round][P][DF_FT]
    if (alive) {  // h of every pair into shared memory, and per (pair, block) the sum of its 32 h
        for (int it = tid; it < P * nblk_d; it += DF_THREADS) {
            const int p = it / nblk_d, j = it % nblk_d;
            const uint4* src = reinterpret_cast<const uint4*>(a.hB + (size_t)p * I + j * 32);
            uint4 v[4];
#pragma unroll
            for (int z = 0; z < 4; ++z) v[z] = __ldcg(src + z);  // written by other CTAs: read at L2
            uint4* dst = reinterpret_cast<uint4*>(hs + (size_t)p * pl.hs_stride + j * 64);
            float sum = 0.f;
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                dst[z] = v[z];
                const uint32_t wd[4] = {v[z].x, v[z].y, v[z].z, v[z].w};
#pragma unroll
                for (int y = 0; y < 4; ++y) sum += __uint_as_float(wd[y] << 16) + __uint_as_float(wd[y] & 0xffff0000u);
            }
            hsum[it] = sum;
        }
        __syncthreads();
        DF_MARK(11);
    }
    if (alive) {
        const int g = lane >> 2, q = lane & 3;
        for (; s < S; ++s) {
            const int b = s % DF_NBUF;
            if (!mbar_wait(&full[warp * DF_NBUF + b], (uint32_t)(s / DF_NBUF) & 1u, 6, s)) { wok = false; break; }
            const int d = s - nC, rr = d / ndw, ui = warp + DF_WARPS * (d % ndw);
            const int pos0 = rt.u_pos[ui], n = rt.u_n[ui];
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            if (rt.u_sl[ui] >= 0)
                df_compute_d_smem<BD, NBD>(ring + (warp * DF_NBUF + b) * DF_CODE_SLOT,
                                           scr + (warp * DF_NBUF + b) * pl.sc_slot, hs + (size_t)pos0 * pl.hs_stride,
                                           pl.hs_stride, hsum + (size_t)pos0 * nblk_d, n, acc);
            __syncwarp();  // the slot's reads are done: it may be refilled
            if (issued < S) issue(issued++);
#pragma unroll
            for (int z = 0; z < 2; ++z) {  // y for pair columns 2q, 2q+1 (when they exist), features g, g+8
                const int jj = 2 * q + z;
                if (jj < n) {
                    const int pos = pos0 + jj;
                    const float wv = rt.w[rt.perm[pos]];
                    float* yp = ypair + ((size_t)rr * P + pos) * DF_FT;
                    yp[g] = wv * acc[z];
                    yp[g + 8] = wv * acc[2 + z];
                }
            }
        }
        alive = __syncthreads_and(wok) != 0;
        DF_MARK(12);
        if (alive)
            for (int u = tid; u < nftc * T * DF_FT; u += DF_THREADS) {
                const int rr = u / (T * DF_FT), t = (u / DF_FT) % T, fl = u % DF_FT;
                const int f = (cta + rr * G) * DF_FT + fl;
                float sum = 0.f;
                for (int j = 0; j < k; ++j) sum += ypair[((size_t)rr * P + rt.inv[t * k + j]) * DF_FT + fl];
                if (a.residual) sum = bf16_bits_to_f32(a.x[(size_t)t * H + f]) + sum;
                if (a.hout) a.hout[(size_t)t * H + f] = sum;
                else a.out[(size_t)t * H + f] = f32_to_bf16_bits(sum);
            }
    }
    // On an error path, wait (bounded) for this warp's copies still in flight
    // before the CTA's shared memory goes away.
    for (int r = s; r < issued; ++r) mbar_wait(&full[warp * DF_NBUF + r % DF_NBUF], (uint32_t)(r / DF_NBUF) & 1u, 8, r);
    DF_MARK(13);
}
