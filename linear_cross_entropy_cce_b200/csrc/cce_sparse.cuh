// Sparse backward for filtered softmax gradients (CUDA cores).
//
// With the gradient filter on, G = dloss * (p * keep - onehot) keeps only a
// few entries per row ("Cut Your Losses in Large-Vocabulary Language
// Models" research-map entry, §Surprising findings: almost all softmax
// entries vanish; first page §Contribution: those entries carry no
// representable gradient).  When one vocabulary chunk of G holds at most
// `cap` non-zeros (density <= 1/2048), its two contractions are cheaper as
// gathers than as dense tensor-core GEMMs:
//   dE_j  = sum_{i : G_ij != 0} G_ij h_i   (column lists, one warp per
//                                           column and 256-wide slice of D)
//   dH_i += sum_{j : G_ij != 0} G_ij e_j   (row lists, added in the final
//                                           dH pass)
// The G producer emits every non-zero (fp32) of the chunk into the chunk's
// list and counts them; chunks over capacity fall back to the dense tensor
// path, whose slab and masks the producer always writes.  The decision is
// taken on the device per chunk, so the host never synchronises.
#pragma once

#include <cub/block/block_scan.cuh>

#include "cce_ptx.cuh"

namespace cce {

struct NzEntry {  // one non-zero of a chunk of G
  int row;        // compact row
  int col;        // column within the chunk
  float g;
  int pad;
};

// Chunk -> (segment, first walk position) for the row lists.
struct ChunkMap {
  int n_segs;
  int chunk_begin[8];  // first global chunk index of each segment
  int width[8];        // chunk width of each segment
};

__device__ __forceinline__ void chunk_lookup(const ChunkMap& m, int c, int& seg, int& c0) {
  int s = 0;
  while (s + 1 < m.n_segs && c >= m.chunk_begin[s + 1]) ++s;
  seg = s;
  c0 = (c - m.chunk_begin[s]) * m.width[s];
}

constexpr int SCAN_THREADS = 1024;

// Exclusive scan of cnt[0..n) into ptr[0..n] (ptr[n] = total) and cur[0..n);
// single CTA.
__device__ __forceinline__ void block_exclusive_scan(const int* cnt, int n, int* ptr, int* cur) {
  using Scan = cub::BlockScan<int, SCAN_THREADS>;
  __shared__ typename Scan::TempStorage tmp;
  const int per = (n + SCAN_THREADS - 1) / SCAN_THREADS;
  const int lo = threadIdx.x * per, hi = min(n, lo + per);
  int s = 0;
  for (int i = lo; i < hi; ++i) s += cnt[i];
  int off, total;
  Scan(tmp).ExclusiveSum(s, off, total);
  for (int i = lo; i < hi; ++i) {
    ptr[i] = off;
    if (cur) cur[i] = off;
    off += cnt[i];
  }
  if (threadIdx.x == 0) ptr[n] = total;
}

// ---- per chunk: column lists ------------------------------------------
// One CTA: exclusive scan of the per-column counts into col_ptr, then the
// scatter of the chunk's entries into column order.
__global__ void __launch_bounds__(SCAN_THREADS)
    sparse_col_sort_kernel(const int* __restrict__ nz_cnt, int cap, const int* __restrict__ col_cnt,
                           int cv, int* __restrict__ col_ptr, int* __restrict__ col_cur,
                           const NzEntry* __restrict__ list, int2* __restrict__ sorted) {
  const int n = *nz_cnt;
  if (n > cap) return;
  block_exclusive_scan(col_cnt, cv, col_ptr, col_cur);
  __syncthreads();
  for (int e = threadIdx.x; e < n; e += SCAN_THREADS) {
    const NzEntry v = list[e];
    const int pos = atomicAdd(&col_cur[v.col], 1);
    sorted[pos] = make_int2(v.row, __float_as_int(v.g));
  }
}

struct SparseDEParams {
  const int* nz_cnt;
  int cap;
  const int* col_ptr;
  const int2* sorted;
  const __nv_bfloat16* Hc;  // [Npad, D]
  int D, cv, c0;
  const int* perm_seg;
  void* dE;
  __nv_bfloat16* dE_comp;
  int mode;  // 0 bf16, 1 fp32 (no Kahan on this path)
};

// Adds g * (8 bf16 at src) into acc.
__device__ __forceinline__ void fma8(float (&acc)[8], float g, const uint4 h) {
  acc[0] = fmaf(g, bf16lo(h.x), acc[0]);
  acc[1] = fmaf(g, bf16hi(h.x), acc[1]);
  acc[2] = fmaf(g, bf16lo(h.y), acc[2]);
  acc[3] = fmaf(g, bf16hi(h.y), acc[3]);
  acc[4] = fmaf(g, bf16lo(h.z), acc[4]);
  acc[5] = fmaf(g, bf16hi(h.z), acc[5]);
  acc[6] = fmaf(g, bf16lo(h.w), acc[6]);
  acc[7] = fmaf(g, bf16hi(h.w), acc[7]);
}

// acc += sum over the n gathered rows of g_k * row_k[d0 .. d0+8): the warp
// holds up to 32 (pointer, g) pairs, one per lane; gathers run 4 deep.  n
// must be the same in every lane (all lanes take part in the shuffles); a
// lane whose slice lies past D passes d0 = 0 and discards its result.
__device__ __forceinline__ void gather_rows_fma(float (&acc)[8], const __nv_bfloat16* myrow, float myg,
                                                int n, int d0) {
  int k = 0;
  for (; k + 4 <= n; k += 4) {
    const __nv_bfloat16* r0 = (const __nv_bfloat16*)__shfl_sync(0xffffffffu, (unsigned long long)myrow, k);
    const __nv_bfloat16* r1 = (const __nv_bfloat16*)__shfl_sync(0xffffffffu, (unsigned long long)myrow, k + 1);
    const __nv_bfloat16* r2 = (const __nv_bfloat16*)__shfl_sync(0xffffffffu, (unsigned long long)myrow, k + 2);
    const __nv_bfloat16* r3 = (const __nv_bfloat16*)__shfl_sync(0xffffffffu, (unsigned long long)myrow, k + 3);
    const float g0 = __shfl_sync(0xffffffffu, myg, k), g1 = __shfl_sync(0xffffffffu, myg, k + 1);
    const float g2 = __shfl_sync(0xffffffffu, myg, k + 2), g3 = __shfl_sync(0xffffffffu, myg, k + 3);
    const uint4 h0 = __ldg(reinterpret_cast<const uint4*>(r0 + d0));
    const uint4 h1 = __ldg(reinterpret_cast<const uint4*>(r1 + d0));
    const uint4 h2 = __ldg(reinterpret_cast<const uint4*>(r2 + d0));
    const uint4 h3 = __ldg(reinterpret_cast<const uint4*>(r3 + d0));
    fma8(acc, g0, h0);
    fma8(acc, g1, h1);
    fma8(acc, g2, h2);
    fma8(acc, g3, h3);
  }
  for (; k < n; ++k) {
    const __nv_bfloat16* r0 = (const __nv_bfloat16*)__shfl_sync(0xffffffffu, (unsigned long long)myrow, k);
    const float g0 = __shfl_sync(0xffffffffu, myg, k);
    fma8(acc, g0, __ldg(reinterpret_cast<const uint4*>(r0 + d0)));
  }
}

// One warp per (column, 256-wide slice of D): the column's entries are
// staged 32 at a time in the lanes (row pointer, g) and gathered 4 deep;
// lane owns 8 consecutive d.  Hot columns (a frequent target collects many
// one-hot entries) keep one warp per slice busy, not one warp per column.
__global__ void sparse_de_kernel(const SparseDEParams p) {
  if (*p.nz_cnt > p.cap) return;
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int nds = (p.D + 255) >> 8;
  for (int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < p.cv * nds; w += nw) {
    const int col = w / nds;
    const int d0 = (w - col * nds) * 256 + lane * 8;
    const int e0 = p.col_ptr[col], e1 = p.col_ptr[col + 1];
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int eb = e0; eb < e1; eb += 32) {
      const int n = min(32, e1 - eb);
      const __nv_bfloat16* myrow = p.Hc;
      float myg = 0.f;
      if (lane < n) {
        const int2 v = p.sorted[eb + lane];
        myrow = p.Hc + (size_t)v.x * p.D;
        myg = __int_as_float(v.y);
      }
      gather_rows_fma(acc, myrow, myg, n, d0 < p.D ? d0 : 0);
    }
    if (d0 >= p.D) continue;
    const int wpos = p.c0 + col;
    const size_t off = (size_t)(p.perm_seg ? p.perm_seg[wpos] : wpos) * p.D + d0;
    if (p.mode == 1) {
      float4* d = reinterpret_cast<float4*>(static_cast<float*>(p.dE) + off);
      d[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      d[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dE) + off) =
          make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]),
                     pack_bf16(acc[4], acc[5]), pack_bf16(acc[6], acc[7]));
    }
  }
}

// ---- after all chunks: row lists for dH ------------------------------------
struct SparseRowsParams {
  const int* nz_cnt;  // [nch]
  int nch, cap;
  const NzEntry* lists;  // [nch][cap]
  int* row_cnt;          // [Npad]
  int* row_cur;
  int2* rsorted;         // (segment << 29 | walk position, g); segments < 2^29 rows
  ChunkMap cmap;
};

__global__ void sparse_row_count_kernel(const SparseRowsParams p) {
  const long long total = (long long)p.nch * p.cap;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(i / p.cap), e = (int)(i - (long long)c * p.cap);
    const int n = p.nz_cnt[c];
    if (n > p.cap || e >= n) continue;
    atomicAdd(&p.row_cnt[p.lists[i].row], 1);
  }
}

__global__ void __launch_bounds__(SCAN_THREADS)
    sparse_row_scan_kernel(const int* __restrict__ row_cnt, int n, int* __restrict__ row_ptr,
                           int* __restrict__ row_cur) {
  block_exclusive_scan(row_cnt, n, row_ptr, row_cur);
}

__global__ void sparse_row_scatter_kernel(const SparseRowsParams p) {
  const long long total = (long long)p.nch * p.cap;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(i / p.cap), e = (int)(i - (long long)c * p.cap);
    const int n = p.nz_cnt[c];
    if (n > p.cap || e >= n) continue;
    const NzEntry v = p.lists[i];
    int seg, c0;
    chunk_lookup(p.cmap, c, seg, c0);
    const int pos = atomicAdd(&p.row_cur[v.row], 1);
    p.rsorted[pos] = make_int2((int)(((unsigned)seg << 29) | (unsigned)(c0 + v.col)),
                               __float_as_int(v.g));
  }
}

}  // namespace cce
