// permute.cu -- group the token->expert assignments by expert.
//
// The fused MoE kernels sort the tokens by expert and group them before the
// grouped GEMM (vLLM fused-MoE page, section 02); FlashMoE (section 5.3) pads
// each group in place to the 128-row tile.  Here the groups stay unpadded and
// a tile list of 128-row blocks per group drives the GEMMs, whose epilogues
// mask the rows past a group's end.
//
// Result: a stable counting sort of the flat assignment list f = t*k + j by
// expert, computed in three deterministic passes over fixed chunks of the list
// (no floating point, no order-dependent atomics in any output):
//   count   per-chunk expert histogram
//   scan    per-expert exclusive scan over chunks, exclusive scan over experts
//           -> expert_offsets, each chunk's base row per expert, the tile list;
//           also resets the grouped GEMMs' work-claim counters
//   scatter each entry's rank among equal experts earlier in its chunk (warp
//           match + per-warp counts) -> sorted_to_flat / flat_to_sorted
#include "moe_internal.h"
#include "pdl.cuh"

namespace moe {
namespace {

__device__ __forceinline__ void record_status(int32_t *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

__global__ void perm_count_kernel(const int32_t *__restrict__ idx, int A, int E, int chunk,
                                  int32_t *__restrict__ blk_cnt, int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ int hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int f0 = blockIdx.x * chunk;
    const int f1 = min(f0 + chunk, A);
    for (int f = f0 + threadIdx.x; f < f1; f += blockDim.x) {
        const int e = idx[f];
        if (e >= 0 && e < E)
            atomicAdd(&hist[e], 1);
        else
            record_status(status, MOE_ERR_BAD_INDEX);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) blk_cnt[(size_t)blockIdx.x * E + e] = hist[e];
}

// Exclusive scan of one value per thread over a block of 1024 threads.
__device__ int block_exclusive_scan(int v, int *warp_tot, int &total)
{
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += o;
        }
        warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
        if (lane == 31) warp_tot[32] = wi;
    }
    __syncthreads();
    const int res = warp_tot[warp] + inc - v;
    total = warp_tot[32];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(1024)
perm_scan_kernel(int E, int nb, const int32_t *__restrict__ blk_cnt, int32_t *__restrict__ blk_base,
                 int32_t *__restrict__ offsets, int32_t *__restrict__ tiles,
                 int32_t *__restrict__ ntiles, int32_t *counters, int ncounters, int32_t *__restrict__ tiles2,
                 int32_t *__restrict__ ntiles2)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int warp_tot[33];
    const int e = threadIdx.x;
    int cnt = 0;
    if (e < E) {
        for (int b = 0; b < nb; ++b) {
            const int c = blk_cnt[(size_t)b * E + e];
            blk_base[(size_t)b * E + e] = cnt;
            cnt += c;
        }
    }
    int total_rows = 0, total_tiles = 0;
    const int off = block_exclusive_scan(cnt, warp_tot, total_rows);
    const int nt = (cnt + kTileRows - 1) / kTileRows;
    const int tstart = block_exclusive_scan(nt, warp_tot, total_tiles);
    // pair tiles of 2 x 128 rows for the 2-CTA GEMMs (optional)
    int total_pairs = 0;
    const int np = (cnt + 2 * kTileRows - 1) / (2 * kTileRows);
    const int pstart = tiles2 ? block_exclusive_scan(np, warp_tot, total_pairs) : 0;
    if (tiles2 && e < E)
        for (int m = 0; m < np; ++m) {
            int32_t *tl = tiles2 + 3 * (size_t)(pstart + m);
            tl[0] = e;
            tl[1] = off + m * 2 * kTileRows;
            tl[2] = min(2 * kTileRows, cnt - m * 2 * kTileRows);
        }
    if (e < E) {
        offsets[e] = off;
        for (int b = 0; b < nb; ++b) blk_base[(size_t)b * E + e] += off;
        for (int m = 0; m < nt; ++m) {
            int32_t *tl = tiles + 3 * (size_t)(tstart + m);
            tl[0] = e;
            tl[1] = off + m * kTileRows;
            tl[2] = min(kTileRows, cnt - m * kTileRows);
        }
    }
    if (threadIdx.x == 0) {
        offsets[E] = total_rows;
        *ntiles = total_tiles;
        if (ntiles2) *ntiles2 = total_pairs;
    }
    if (counters && threadIdx.x < ncounters) counters[threadIdx.x] = 0;
}

__global__ void perm_scatter_kernel(const int32_t *__restrict__ idx, int A, int E,
                                    const int32_t *__restrict__ blk_base, int32_t *__restrict__ s2f,
                                    int32_t *__restrict__ f2s)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ int wcnt[];  // [warps][E]: entries of each expert in each warp
    const int nw = blockDim.x / 32;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int i = threadIdx.x; i < nw * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const int f = blockIdx.x * blockDim.x + threadIdx.x;
    const int e = f < A ? idx[f] : -1;
    const bool valid = e >= 0 && e < E;
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
    const unsigned lower = (1u << lane) - 1u;
    const int rank = __popc(peers & lower);
    if (valid && rank == 0) wcnt[warp * E + e] = __popc(peers);
    __syncthreads();
    if (!valid) return;
    int prior = 0;
    for (int w = 0; w < warp; ++w) prior += wcnt[w * E + e];
    const int pos = blk_base[(size_t)blockIdx.x * E + e] + prior + rank;
    s2f[pos] = f;
    f2s[f] = pos;
}

// x rows into expert-sorted order, a warp per assignment in flat order: warp f
// copies x[f / k] to xs[f2s[f]].  The k copies of a token are made by neighbouring
// warps, close in time, so x is read from DRAM about once; walking the sorted rows
// instead reads each x row k times far apart, and the copy's own write stream evicts
// x from L2 in between.
__global__ void gather_rows_kernel(const __nv_bfloat16 *__restrict__ x,
                                   const int32_t *__restrict__ f2s, int A, int H, int k,
                                   __nv_bfloat16 *__restrict__ xs)
{
    pdl_wait();
    pdl_trigger();
    const int f = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (f >= A) return;
    const int pos = f2s[f];
    if ((unsigned)pos >= (unsigned)A) return;  // never outside xs
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)(f / k) * H);
    uint4 *dst = reinterpret_cast<uint4 *>(xs + (size_t)pos * H);
    for (int c = lane; c < H / 8; c += 32) dst[c] = src[c];
}

}  // namespace

cudaError_t launch_permute(const moe_dims_t &d, const WsLayout &L, const int32_t *idx,
                           int32_t *blk_cnt, int32_t *blk_base, int32_t *offsets, int32_t *s2f,
                           int32_t *f2s, int32_t *tiles, int32_t *ntiles, WsHeader *hdr,
                           cudaStream_t st, int32_t *tiles2, int32_t *ntiles2)
{
    const int A = d.T * d.top_k, E = d.E;
    cudaError_t e = launch_pdl(perm_count_kernel, dim3(L.nb), dim3(256), E * sizeof(int), st, idx, A, E, L.chunk,
                               blk_cnt, hdr ? &hdr->status : nullptr);
    if (e == cudaSuccess)
        e = launch_pdl(perm_scan_kernel, dim3(1), dim3(1024), 0, st, E, L.nb, blk_cnt, blk_base, offsets, tiles,
                       ntiles, hdr ? hdr->counter : nullptr, hdr ? 7 : 0, tiles2, ntiles2);
    if (e == cudaSuccess)
        e = launch_pdl(perm_scatter_kernel, dim3(L.nb), dim3(L.chunk), (size_t)(L.chunk / 32) * E * sizeof(int), st,
                       idx, A, E, blk_base, s2f, f2s);
    return e;
}

cudaError_t launch_gather_rows(const __nv_bfloat16 *x, const int32_t *f2s, int T, int H, int top_k,
                               __nv_bfloat16 *xs, cudaStream_t st)
{
    const int A = T * top_k, rows_per_block = 8;
    return launch_pdl(gather_rows_kernel, dim3((A + rows_per_block - 1) / rows_per_block), dim3(rows_per_block * 32),
                      0, st, x, f2s, A, H, top_k, xs);
}

}  // namespace moe
