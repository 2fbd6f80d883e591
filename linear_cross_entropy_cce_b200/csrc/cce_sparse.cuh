// Sparse backward for filtered softmax gradients (CUDA cores).
//
// With the gradient filter on, G = dloss * (p * keep - onehot) keeps only a
// few entries per row ("Cut Your Losses in Large-Vocabulary Language
// Models" research-map entry, §Surprising findings: almost all softmax
// entries vanish; first page §Contribution: those entries carry no
// representable gradient).  When one vocabulary chunk of G holds at most
// `cap` non-zeros (density <= 1/2048), its two contractions are cheaper as
// gathers than as dense tensor-core GEMMs:
//   dE_j  = sum_{i : G_ij != 0} G_ij h_i   (column lists over H_c rows)
//   dH_i += sum_{j : G_ij != 0} G_ij e_j   (row lists over E rows)
// The G producer emits every non-zero (fp32) of a chunk into the chunk's
// list; chunks over capacity take the dense tensor path instead.  The
// decision is taken on the device per chunk, so the host never synchronises.
//
// Both contractions run once, after every chunk's G is known:
//   sparse_count_kernel    entries per column (global walk position) and row
//   (exclusive scans)      column and row offsets (CSR)
//   sparse_scatter_kernel  entries into column order and into row order
//   csr_rows_kernel<DERows>  each dE row of a sparse chunk: the gather over
//                            its column list (zero when empty)
//   csr_rows_kernel<DHRows>  each valid dH row: the dense accumulator plus
//                            the gather over its row list; dh_fill_kernel
//                            writes the other rows
// Entries of one row or column are summed in an order set by atomics, so
// these sums are not bitwise reproducible run to run.
#pragma once

#include <type_traits>

#include "cce_ptx.cuh"

namespace cce {

struct NzEntry {  // one non-zero of a chunk of G
  int row;        // compact row
  int col;        // column within the chunk
  float g;
  int pad;
};

constexpr int SP_MAX_SEGS = 8;

// Chunk -> (segment, first walk position) for the sparse lists.
struct ChunkMap {
  int n_segs;
  int chunk_begin[SP_MAX_SEGS];  // first global chunk index of each segment
  int width[SP_MAX_SEGS];        // chunk width of each segment
  int live_off[SP_MAX_SEGS];     // first global walk position of each segment
};

__device__ __forceinline__ void chunk_lookup(const ChunkMap& m, int c, int& seg, int& c0) {
  int s = 0;
  while (s + 1 < m.n_segs && c >= m.chunk_begin[s + 1]) ++s;
  seg = s;
  c0 = (c - m.chunk_begin[s]) * m.width[s];
}

// ---- lists -> CSR ------------------------------------------------------------
struct SparseListParams {
  const int* nz_cnt;  // [nch] entries emitted per chunk; > cap: dense chunk, list unused
  int nch, cap;
  const NzEntry* lists;  // [nch][cap]
  ChunkMap cmap;
  int* col_cnt;          // [V_live + 1] entries per global walk position; null: no dE lists
  const int* col_ptr;    // [V_live + 1] exclusive scan of col_cnt
  int2* csorted;         // (compact row, g) in column order
  int* row_cnt;          // [Npad + 1] entries per compact row
  const int* row_ptr;    // [Npad + 1]
  int2* rsorted;         // (segment << 29 | walk position in segment, g) in row order
};

// grid.y = chunk; grid.x strides over the chunk's entries.
__global__ void sparse_count_kernel(const SparseListParams p) {
  const int c = blockIdx.y;
  const int n = p.nz_cnt[c];
  if (n > p.cap) return;
  int seg, c0;
  chunk_lookup(p.cmap, c, seg, c0);
  const int gbase = p.cmap.live_off[seg] + c0;
  const NzEntry* list = p.lists + (size_t)c * p.cap;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    const NzEntry v = list[e];
    if (p.col_cnt) atomicAdd(&p.col_cnt[gbase + v.col], 1);
    atomicAdd(&p.row_cnt[v.row], 1);
  }
}

// Places every entry at offset + (its count, decremented): the counts end at 0.
__global__ void sparse_scatter_kernel(const SparseListParams p) {
  const int c = blockIdx.y;
  const int n = p.nz_cnt[c];
  if (n > p.cap) return;
  int seg, c0;
  chunk_lookup(p.cmap, c, seg, c0);
  const int gbase = p.cmap.live_off[seg] + c0;
  const NzEntry* list = p.lists + (size_t)c * p.cap;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    const NzEntry v = list[e];
    const int gv = __float_as_int(v.g);
    if (p.col_cnt) {
      const int gw = gbase + v.col;
      p.csorted[p.col_ptr[gw] + atomicSub(&p.col_cnt[gw], 1) - 1] = make_int2(v.row, gv);
    }
    p.rsorted[p.row_ptr[v.row] + atomicSub(&p.row_cnt[v.row], 1) - 1] =
        make_int2((int)(((unsigned)seg << 29) | (unsigned)(c0 + v.col)), gv);
  }
}

// ---- CSR x dense rows ----------------------------------------------------------
constexpr int GATHER_STAGE = 512;  // list entries staged in shared memory at once
constexpr int GATHER_RANGE = 64;   // most output rows one block takes at a time
constexpr int GATHER_MAX_THREADS = 512;

struct GatherSrc {
  const __nv_bfloat16* src;
  float g;
  int row;  // output row within the block's range
};

// Adds g * (8 bf16 in h) into acc.
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

__device__ __forceinline__ void store_row8(void* row, int d, const float (&a)[8], int fp32_out) {
  if (fp32_out) {
    float4* o = reinterpret_cast<float4*>(static_cast<float*>(row) + d);
    o[0] = make_float4(a[0], a[1], a[2], a[3]);
    o[1] = make_float4(a[4], a[5], a[6], a[7]);
  } else {
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(row) + d) =
        make_uint4(pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]), pack_bf16(a[4], a[5]),
                   pack_bf16(a[6], a[7]));
  }
}

// Rows of a CSR matrix times dense bf16 source rows, one output row each:
//   out_r = addend_r + sum_{e in [ptr[r], ptr[r+1])} g_e * src(key_e).
// A block takes `range` consecutive rows: their list entries are contiguous,
// so it stages them (window by window) with each entry's row and walks them
// in one flat pass, 8 source loads in flight across row boundaries; a row is
// stored when the walk passes it, empty rows included.  Each thread owns 8
// consecutive elements of D (a slice of blockDim * 8 at a time).
//
// R supplies: rows() (count), ptr, ent, src(key), out(row) (null: not
// written here), addend(row) (null: 0), fp32_out, D, range.  For DHRows the
// addend (dH_acc) is read only when some chunk took the dense route.

// dE rows of the chunks taken by the sparse route, indexed by global walk
// position w (segment s, w - live_off[s] within it).  Rows of dense chunks are
// left to the dense contraction.
struct DERows {
  const int* ptr;  // [V_live + 1]
  const int2* ent; // (compact row, g)
  const __nv_bfloat16* Hc;  // [Npad, D]
  long long v_live;
  int D, range;
  const int* nz_cnt;
  int cap;
  ChunkMap cmap;
  const int* vocab_perm;  // concatenated per-segment permutations, or null
  void* dE[SP_MAX_SEGS];
  int fp32_out;

  __device__ long long rows() const { return v_live; }
  __device__ const __nv_bfloat16* src(int key) const { return Hc + (size_t)key * D; }
  __device__ void* out(long long r) const {
    const int w = (int)r;
    int s = 0;
    while (s + 1 < cmap.n_segs && w >= cmap.live_off[s + 1]) ++s;
    const int wl = w - cmap.live_off[s];
    if (nz_cnt[cmap.chunk_begin[s] + wl / cmap.width[s]] > cap) return nullptr;
    const size_t row = (size_t)(vocab_perm ? vocab_perm[w] : wl);
    return fp32_out ? (void*)(static_cast<float*>(dE[s]) + row * D)
                    : (void*)(static_cast<__nv_bfloat16*>(dE[s]) + row * D);
  }
  __device__ const float* addend(long long) const { return nullptr; }
  static constexpr bool kAddend = false;  // rows start from zero
};

// dH rows of the valid (compact) rows j: dH_acc row j (when some chunk took
// the dense route) plus the row list over E rows, written to original row
// idx[j].  Ignored and bad-target rows are written by dh_fill_kernel.
struct DHRows {
  const int* ptr;   // [Npad + 1]; null: no row lists (every chunk dense)
  const int2* ent;  // (segment << 29 | walk position in segment, g)
  const int* n_valid;
  const int* idx;   // compact -> original row
  const float* dH_acc;  // [Npad, D]; read only when some chunk took the dense route
  const int* nz_cnt;  // [nch]; null: every chunk took the dense route
  int nch, cap;
  int D, range;
  void* dH;
  int fp32_out;
  const __nv_bfloat16* E[SP_MAX_SEGS];
  int live_off[SP_MAX_SEGS];
  const int* vocab_perm;

  __device__ long long rows() const { return *n_valid; }
  __device__ const __nv_bfloat16* src(int key) const {
    const int s = (int)((unsigned)key >> 29), w = key & ((1 << 29) - 1);
    const int loc = vocab_perm ? vocab_perm[live_off[s] + w] : w;
    return E[s] + (size_t)loc * D;
  }
  __device__ void* out(long long j) const {
    const size_t i = (size_t)idx[j];
    return fp32_out ? (void*)(static_cast<float*>(dH) + i * D)
                    : (void*)(static_cast<__nv_bfloat16*>(dH) + i * D);
  }
  __device__ const float* addend(long long j) const { return dH_acc + (size_t)j * D; }
  static constexpr bool kAddend = true;  // dH_acc, when some chunk was dense
};

// FP32: the output rows are fp32 (else bf16), fixed per launch.
template <class R, bool FP32>
__global__ void __launch_bounds__(GATHER_MAX_THREADS, 1) csr_rows_kernel(const R p) {
  __shared__ int sp[GATHER_RANGE + 1];
  __shared__ void* dst[GATHER_RANGE];
  __shared__ const float* add[GATHER_RANGE];
  __shared__ GatherSrc stage[GATHER_STAGE];
  bool use_add = true;
  if constexpr (std::is_same<R, DHRows>::value) {
    // dH_acc holds anything only if some chunk took the dense route
    __shared__ int dense_any;
    if (threadIdx.x == 0) dense_any = p.nz_cnt ? 0 : 1;
    __syncthreads();
    if (p.nz_cnt)
      for (int c = threadIdx.x; c < p.nch; c += blockDim.x)
        if (p.nz_cnt[c] > p.cap) dense_any = 1;
    __syncthreads();
    use_add = dense_any != 0;
  }
  const long long nrows = p.rows();
  const long long step = (long long)gridDim.x * p.range;
  for (long long r0 = (long long)blockIdx.x * p.range; r0 < nrows; r0 += step) {
    const int nr = (int)min((long long)p.range, nrows - r0);
    __syncthreads();  // the previous range is no longer read
    for (int k = threadIdx.x; k <= nr; k += blockDim.x) {
      sp[k] = p.ptr ? p.ptr[r0 + k] : 0;
      if (k < nr) {
        dst[k] = p.out(r0 + k);
        add[k] = use_add ? p.addend(r0 + k) : nullptr;
      }
    }
    __syncthreads();
    const int E0 = sp[0], E1 = sp[nr];
    for (int db = 0; db < p.D; db += blockDim.x * 8) {
      const int d = db + threadIdx.x * 8;
      const bool act = d < p.D;
      int cur = 0;  // row being accumulated
      float a[8];
      bool touched = false;  // the current row has an entry (or an addend)
      auto start = [&](int r) {
        touched = false;
        const float* ad = R::kAddend ? add[r] : nullptr;
        if (ad && act) {
          touched = true;
          const float4 u = *reinterpret_cast<const float4*>(ad + d);
          const float4 v = *reinterpret_cast<const float4*>(ad + d + 4);
          a[0] = u.x; a[1] = u.y; a[2] = u.z; a[3] = u.w;
          a[4] = v.x; a[5] = v.y; a[6] = v.z; a[7] = v.w;
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) a[k] = 0.f;
        }
      };
      auto finish = [&](int r) {
        if (!act || !dst[r]) return;
        if (touched) {
          store_row8(dst[r], d, a, FP32);
        } else if (FP32) {  // an empty row: zeros, nothing to convert
          float4* o = reinterpret_cast<float4*>(static_cast<float*>(dst[r]) + d);
          o[0] = make_float4(0.f, 0.f, 0.f, 0.f);
          o[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dst[r]) + d) = make_uint4(0u, 0u, 0u, 0u);
        }
      };
      start(0);
      for (int wb = E0; wb < E1; wb += GATHER_STAGE) {
        const int n = min(GATHER_STAGE, E1 - wb);
        __syncthreads();  // the previous window is no longer read
        for (int k = threadIdx.x; k < n; k += blockDim.x) {
          const int e = wb + k;
          int lo = 0, hi = nr;  // the row r with sp[r] <= e < sp[r + 1]
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (sp[mid] <= e) lo = mid; else hi = mid;
          }
          const int2 v = p.ent[e];
          stage[k] = GatherSrc{p.src(v.x), __int_as_float(v.y), lo};
        }
        __syncthreads();
        if (!act) continue;
        int k = 0;
        for (; k + 8 <= n; k += 8) {
          uint4 h[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) h[u] = __ldg(reinterpret_cast<const uint4*>(stage[k + u].src + d));
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int r = stage[k + u].row;
            while (cur < r) {
              finish(cur);
              start(++cur);
            }
            fma8(a, stage[k + u].g, h[u]);
            touched = true;
          }
        }
        for (; k < n; ++k) {
          const int r = stage[k].row;
          while (cur < r) {
            finish(cur);
            start(++cur);
          }
          fma8(a, stage[k].g, __ldg(reinterpret_cast<const uint4*>(stage[k].src + d)));
          touched = true;
        }
      }
      // the rows after the last entry (all of them if the range has none)
      for (;;) {
        finish(cur);
        if (++cur >= nr) break;
        start(cur);
      }
    }
  }
}

// dH rows without a compact row: 0 for ignored rows, NaN for bad targets.
__global__ void dh_fill_kernel(const int* __restrict__ pos_of_row, long long N, int D, void* dH,
                               int fp32_out) {
  const int per_row = D / 8;
  const long long total = N * per_row;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const long long i = t / per_row;
    const int j = pos_of_row[i];
    if (j >= 0) continue;
    const float f = j == -1 ? 0.f : __int_as_float(0x7fc00000);
    const float a[8] = {f, f, f, f, f, f, f, f};
    void* row = fp32_out ? (void*)(static_cast<float*>(dH) + i * D)
                         : (void*)(static_cast<__nv_bfloat16*>(dH) + i * D);
    store_row8(row, (int)(t - i * per_row) * 8, a, fp32_out);
  }
}

// Rows per block range: enough ranges for every block, at most GATHER_RANGE.
inline int gather_range(long long rows, int blocks) {
  const long long r = rows / (blocks > 0 ? blocks : 1);
  return (int)(r < 4 ? 4 : (r > GATHER_RANGE ? GATHER_RANGE : r));
}

// Threads per block for the gathers: 8 elements of D each, whole warps.
inline int gather_threads(long long D) {
  const long long t = ((D / 8 + 31) / 32) * 32;
  return (int)(t < GATHER_MAX_THREADS ? t : GATHER_MAX_THREADS);
}

}  // namespace cce
