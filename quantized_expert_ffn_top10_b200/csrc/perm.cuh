// Grouping of (token, slot) pairs by expert, the routing-count histogram and
// the prefill tile list.
//
// Pair p = t*k + j routes token t to expert idx[p].  counts[e] is the number of
// pairs on e, offsets the exclusive prefix sum, perm the pairs grouped by
// expert with ascending p inside a group (a stable counting sort), and
// inv[perm[i]] = i.  Three passes: per-chunk counts (shared-memory counters,
// order independent), one block that scans them, and a scatter in which each
// chunk's warps take their turn so that ranks follow p.
#pragma once
#include "common.cuh"

#define PERM_CHUNK 1024
#define PREFILL_TILE_N 192  // max tokens per grouped-GEMM tile

struct PermArgs {
    const int32_t* idx;   // [P]
    int P, E, nchunks;
    int32_t* chunk_cnt;   // [nchunks][E] counts, then absolute bases
    int32_t* offsets;     // [E+1]
    int32_t* perm;        // [P]
    int32_t* inv;         // [P]
    int32_t* uniq;        // [E] experts with pairs, ascending
    int32_t* meta;        // [0] = number of such experts, [1] = number of prefill tiles
    int4* tiles;          // [max tiles] (expert, first row, rows, 0) or null
    uint32_t* hist;       // [L][E] or null
    int layer;
};

// Expert of pair p.  The top-k only writes valid experts; an index outside
// [0, E) would mean a library fault, and is counted as expert 0 (the same in
// both passes, so the grouping stays a bijection) with MOE_ERR_RANGE latched.
__device__ __forceinline__ int pair_expert(const PermArgs& a, int p) {
    const int e = a.idx[p];
    if ((unsigned)e < (unsigned)a.E) return e;
    moe_set_status(MOE_ERR_RANGE);
    return 0;
}

__global__ void __launch_bounds__(PERM_CHUNK) k_perm_count(PermArgs a) {
    __shared__ int cnt[MOE_MAX_E];
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    int p = blockIdx.x * PERM_CHUNK + threadIdx.x;
    if (p < a.P) atomicAdd(&cnt[pair_expert(a, p)], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.chunk_cnt[(size_t)blockIdx.x * a.E + e] = cnt[e];
}

// exclusive scan over the block (blockDim.x == MOE_MAX_E); returns the total
__device__ __forceinline__ int block_excl_scan(int v, int* excl, int* s_warp) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    __syncthreads();
    if (lane == 31) s_warp[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int w = lane < nw ? s_warp[lane] : 0, wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < nw) s_warp[lane] = wi - w;  // exclusive warp base
        if (lane == nw - 1) s_warp[32] = wi;   // total
    }
    __syncthreads();
    *excl = s_warp[wid] + incl - v;
    int total = s_warp[32];
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(MOE_MAX_E) k_perm_scan(PermArgs a) {
    __shared__ int s_warp[33];
    const int e = threadIdx.x;
    int c = 0;
    if (e < a.E)
        for (int b0 = 0; b0 < a.nchunks; b0 += 16) {  // 16 loads in flight, then their bases
            int v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = b0 + j < a.nchunks ? a.chunk_cnt[(size_t)(b0 + j) * a.E + e] : 0;
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (b0 + j < a.nchunks) {
                    a.chunk_cnt[(size_t)(b0 + j) * a.E + e] = c;  // relative base of chunk b0 + j
                    c += v[j];
                }
        }
    int off;
    int total = block_excl_scan(c, &off, s_warp);
    if (e < a.E) {
        a.offsets[e] = off;  // chunk b of expert e starts at offsets[e] + chunk_cnt[b][e]
        if (a.hist) a.hist[(size_t)a.layer * a.E + e] += (uint32_t)c;
    }
    if (e == 0) a.offsets[a.E] = total;
    int upos;
    int nuniq = block_excl_scan((e < a.E && c > 0) ? 1 : 0, &upos, s_warp);
    if (e < a.E && c > 0) a.uniq[upos] = e;
    int nt = (e < a.E && c > 0) ? (c + PREFILL_TILE_N - 1) / PREFILL_TILE_N : 0;
    int tpos;
    int ntiles = block_excl_scan(nt, &tpos, s_warp);
    if (a.tiles && nt > 0) {
        // split the expert's rows into nt tiles of near-equal size
        int per = (c + nt - 1) / nt;
        for (int i = 0; i < nt; ++i) {
            int r0 = i * per, n = min(per, c - r0);
            a.tiles[tpos + i] = make_int4(e, off + r0, n, 0);
        }
    }
    if (e == 0) {
        a.meta[0] = nuniq;
        a.meta[1] = ntiles;
    }
}

__global__ void __launch_bounds__(PERM_CHUNK) k_perm_scatter(PermArgs a) {
    __shared__ int cursor[MOE_MAX_E];
    for (int e = threadIdx.x; e < a.E; e += blockDim.x)
        cursor[e] = a.offsets[e] + a.chunk_cnt[(size_t)blockIdx.x * a.E + e];
    __syncthreads();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int p = blockIdx.x * PERM_CHUNK + threadIdx.x;
    const bool valid = p < a.P;
    const int e = valid ? pair_expert(a, p) : -1;
    const unsigned grp = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(grp & ((1u << lane) - 1));
    const int leader = __ffs(grp) - 1;
    for (int w = 0; w < (PERM_CHUNK >> 5); ++w) {
        if (wid == w && valid) {
            int pos = cursor[e] + rank;
            a.perm[pos] = p;
            a.inv[p] = pos;
        }
        __syncwarp();
        if (wid == w && valid && lane == leader) cursor[e] += __popc(grp);
        __syncthreads();
    }
}

// hist[layer][e] += offsets[e+1] - offsets[e]; one owner thread per expert
__global__ void k_hist_add(const int32_t* __restrict__ offsets, int E, int layer, uint32_t* __restrict__ hist) {
    int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < E) hist[(size_t)layer * E + e] += (uint32_t)(offsets[e + 1] - offsets[e]);
}
