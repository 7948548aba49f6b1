// Token permutation: from the gate's (idx, w) to expert-contiguous rows.
//
// The expert loop of "MoE 前向四步" in the DeepSeek-V3 model.py notes
// (73biji.xyz/llm_pp_dsv3) runs each expert on x[idx]: the tokens that chose it.
// Here those gathers become one deterministic counting sort:
//   counts   per 32-token chunk and expert (written by the gate-select CTAs),
//   scan     per expert over chunks, then over experts -> row offsets, plus the
//            GEMM chunks (shared experts appended as always-selected groups of
//            all T tokens),
//   scatter  rank of (t, j) inside its expert = number of earlier tokens of the
//            same chunk that chose that expert (bit mask + popc), so rows of one
//            expert are in ascending token order; bf16 layers also copy x into
//            the permuted activation buffer. The scatter CTAs also fill the two
//            grouped GEMMs' tile lists, which the one-CTA scan would take tens
//            of microseconds to write for a long prefill.
#include <cuda_bf16.h>

#include <algorithm>

#include "ktmoe_internal.cuh"

namespace ktmoe {
namespace {

constexpr int kScanThreads = 1024;
// Scatter CTA: 16 warps over one 32-token chunk (two tokens' row copies per warp).
constexpr int kScatterThreads = 512;

// Exclusive scan over n <= kScanThreads ints in shared memory; returns total.
__device__ int block_exclusive_scan(int* buf, int n) {
  __shared__ int warp_tot[kScanThreads / 32];
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int v = tid < n ? buf[tid] : 0;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int wv = lane < (int)(blockDim.x / 32) ? warp_tot[lane] : 0;
    int wi = wv;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += o;
    }
    warp_tot[lane] = wi - wv;  // exclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = incl - v + warp_tot[warp];
  __syncthreads();
  if (tid < n) buf[tid] = excl;
  __shared__ int total;
  if (tid == n - 1) total = excl + v;
  __syncthreads();
  return total;
}

// Largest i with base[i] <= v, for a non-decreasing base[0..n] with base[0] = 0.
__device__ __forceinline__ int find_group(const int* base, int n, int v) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (base[mid] <= v) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Tile t of a group with nc chunks and F feature tiles: blocks of kTileBlock
// chunks, feature-tile-major inside a block, so the pairs that run one weight
// tile over several token chunks run together.
__device__ __forceinline__ int2 tile_of(int local, int nc, int F, int chunk0) {
  const int b = local / (kTileBlock * F);
  const int bs = min(kTileBlock, nc - b * kTileBlock);
  const int rem = local - b * kTileBlock * F;
  return make_int2(chunk0 + b * kTileBlock + rem % bs, rem / bs);
}

// Positions of a proportional merge of two tile streams, H (nh tiles) and L
// (nl tiles): element i of a stream of n has key (2i+1)/(2n); keys ascend, H
// first on equal keys. Integer arithmetic, so the positions form a permutation.
__device__ __forceinline__ int merged_pos_h(int i, int nh, int nl) {
  const int64_t A = (int64_t)(2 * i + 1) * nl;           // L tiles with (2j+1)*nh < A go first
  const int64_t M = A > 0 ? (A - 1) / nh : 0;
  const int64_t c = (M + 1) / 2;
  return i + (int)(c < nl ? c : nl);
}
__device__ __forceinline__ int merged_pos_l(int j, int nh, int nl) {
  const int64_t B = (int64_t)(2 * j + 1) * nh;           // H tiles with (2i+1)*nl <= B go first
  const int64_t M = B / nl;
  const int64_t c = (M + 1) / 2;
  return j + (int)(c < nh ? c : nh);
}

// Fill one GEMM's tile list with all threads of the grid: groups with at least
// kHeavyRows rows (compute-bound) form stream H, the others (weight-streaming)
// stream L; each stream is ordered per group by tile_of, and the two are merged
// proportionally so that the pairs running at any moment mix both kinds. cb is
// the groups' first GEMM chunk (cb[NG] = all chunks), hcb / lcb the exclusive
// prefix of their chunks in H / L; F feature tiles per chunk.
__device__ void fill_tiles(int2* __restrict__ tiles, int F, int NG, const int* cb, const int* hcb,
                           const int* lcb, int* err) {
  const int nh = F * hcb[NG], nl = F * lcb[NG];
  const int stride = gridDim.x * gridDim.y * blockDim.x;
  const int t0 = (blockIdx.y * gridDim.x + blockIdx.x) * blockDim.x + threadIdx.x;
  for (int i = t0; i < nh; i += stride) {
    const int g = find_group(hcb, NG, i / F);
    const int pos = merged_pos_h(i, nh, nl);
    if (in_range(pos, 0, nh + nl, err, 104))
      tiles[pos] = tile_of(i - F * hcb[g], cb[g + 1] - cb[g], F, cb[g]);
  }
  for (int j = t0; j < nl; j += stride) {
    const int g = find_group(lcb, NG, j / F);
    const int pos = merged_pos_l(j, nh, nl);
    if (in_range(pos, 0, nh + nl, err, 104))
      tiles[pos] = tile_of(j - F * lcb[g], cb[g + 1] - cb[g], F, cb[g]);
  }
}

__global__ void __launch_bounds__(kScanThreads)
permute_scan_kernel(int E, int S, int T_, int k, int nperm, int Fu, int Fd, int chunk_rows,
                    const __grid_constant__ SlotTable tab, int n_local, int sb, int se,
                    const int32_t* __restrict__ chunk_counts, int32_t* __restrict__ chunk_base,
                    int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                    Chunk* __restrict__ chunks, int32_t* __restrict__ meta,
                    int32_t* __restrict__ gchunk0, int max_chunks, int* __restrict__ err) {
  pdl_wait();
  constexpr int NGMAX = kMaxExperts + kMaxShared;
  __shared__ int tot[NGMAX];
  __shared__ int rows0[NGMAX];
  __shared__ int cb[NGMAX + 1];
  const int tid = threadIdx.x;
  const int NG = E + S;
  // Per-expert totals over the chunks; shared experts hold tokens [sb, se) (all
  // T unless the caller splits them); routed experts computed elsewhere (slot
  // -1) hold none. The chunks of each routed expert are cut into P segments,
  // one thread each (thread e + p*E takes segment p of expert e), so that a
  // long prefill's count loads run P-wide; each thread keeps 8 loads in flight.
  __shared__ int seg[kScanThreads];
  constexpr int kBatch = 8;
  const int P = E > 0 ? max(1, min(32, kScanThreads / E)) : 1;
  const int seg_len = (nperm + P - 1) / P;
  const int se_e = tid % max(E, 1), se_p = tid / max(E, 1);
  const bool seg_thread = E > 0 && se_p < P;
  const int c_lo = min(nperm, se_p * seg_len), c_hi = min(nperm, c_lo + seg_len);
  if (seg_thread) {
    int run = 0;
    if (tab.slot[se_e] >= 0) {
      for (int c0 = c_lo; c0 < c_hi; c0 += kBatch) {
        int v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
          v[u] = c0 + u < c_hi ? chunk_counts[(int64_t)(c0 + u) * E + se_e] : 0;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) run += v[u];
      }
    }
    seg[tid] = run;
  }
  __syncthreads();
  if (tid < NG) {
    int run = 0;
    if (tid >= E) {
      run = se - sb;
    } else {
      for (int q = 0; q < P; ++q) {   // segment sums -> exclusive prefix per segment
        const int v = seg[q * E + tid];
        seg[q * E + tid] = run;
        run += v;
      }
    }
    tot[tid] = run;
    rows0[tid] = run;
    counts[tid] = run;
  }
  __syncthreads();
  // Routed experts: rows [0, T*k); shared expert s: rows T*k + s*T + t.
  const int routed_rows = block_exclusive_scan(rows0, E);
  if (tid >= E && tid < NG) rows0[tid] = T_ * k + (tid - E) * T_;
  __syncthreads();
  if (tid < NG) offsets[tid] = rows0[tid];
  if (tid == 0) offsets[NG] = T_ * k + S * T_;
  // Chunk bases (global row of each permutation chunk's first row per expert),
  // by the same segments.
  if (seg_thread) {
    int run = rows0[se_e] + seg[tid];
    for (int c0 = c_lo; c0 < c_hi; c0 += kBatch) {
      int v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        v[u] = c0 + u < c_hi ? chunk_counts[(int64_t)(c0 + u) * E + se_e] : 0;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (c0 + u < c_hi) chunk_base[(int64_t)(c0 + u) * E + se_e] = run;
        run += v[u];
      }
    }
  }
  // GEMM chunks of chunk_rows rows (their tile lists are the scatter's).
  if (tid < NG) cb[tid] = (tot[tid] + chunk_rows - 1) / chunk_rows;
  __syncthreads();
  const int n_chunks = block_exclusive_scan(cb, NG);
  // (Checked build) more routed rows or chunks than the workspace holds: no
  // GEMM work is scheduled.
  const bool fits = in_range(routed_rows, 0, (int64_t)T_ * k + 1, err, 101) &&
                    in_range(n_chunks, 0, max_chunks + 1, err, 102);
  if (tid < NG) gchunk0[tid] = cb[tid];
  if (tid == 0) {
    cb[NG] = n_chunks;
    meta[0] = fits ? n_chunks : 0;
    meta[1] = fits ? n_chunks * Fu : 0;
    meta[2] = fits ? n_chunks * Fd : 0;
    meta[3] = 0;   // gate/up GEMM tile counter
    meta[4] = 0;   // down GEMM tile counter
  }
  __syncthreads();
  if (!fits) return;
  // The chunks name weight slots: routed expert g in slot tab.slot[g], shared
  // expert E + s in slot n_local + s.
  for (int i = tid; i < n_chunks; i += blockDim.x) {
    const int g = find_group(cb, NG, i);
    const int r = (i - cb[g]) * chunk_rows;
    const int slot = g < E ? tab.slot[g] : n_local + (g - E);
    const int row0 = g < E ? rows0[g] : rows0[g] + sb;
    const int src0 = g < E ? rows0[g] : sb;
    chunks[i] = Chunk{slot, row0 + r, min(chunk_rows, tot[g] - r), src0 + r};
  }
}

// Copy modes of the scatter.
enum { kNoCopy = 0, kCopyBf16 = 1, kCopyF8 = 2 };

template <int kMode>
__global__ void __launch_bounds__(kScatterThreads)
permute_scatter_kernel(int E, int S, int T_, int k, int d, int chunk_rows,
                       const __grid_constant__ SlotTable tab,
                       int sb, int se,
                       const int32_t* __restrict__ idx, const float* __restrict__ w,
                       const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ offsets,
                       const int32_t* __restrict__ gchunk0, int32_t* __restrict__ row_of,
                       int32_t* __restrict__ tok_of, float* __restrict__ row_weight,
                       const uint4* __restrict__ x, uint4* __restrict__ xperm,
                       const uint8_t* __restrict__ xs, uint8_t* __restrict__ tok_sf,
                       int max_chunks, const int32_t* __restrict__ counts,
                       const int32_t* __restrict__ meta, int Fu, int Fd,
                       int2* __restrict__ tiles_up, int2* __restrict__ tiles_dn,
                       int* __restrict__ err) {
  pdl_wait();
  __shared__ uint32_t mask[kMaxExperts];
  __shared__ int srow[kPermChunk * kMaxTopk];
  // The grouped GEMMs' tile lists (none when the scan found that the chunks do
  // not fit the workspace): every CTA builds the groups' chunk prefixes in H and
  // L from the scan's chunk starts and row counts, then fills its share.
  {
    constexpr int NGMAX = kMaxExperts + kMaxShared;
    __shared__ int s_cb[NGMAX + 1], s_hcb[NGMAX + 1], s_lcb[NGMAX + 1];
    const int NG = E + S;
    if (meta[1] > 0) {
      for (int g = threadIdx.x; g < NG; g += blockDim.x) s_cb[g] = gchunk0[g];
      if (threadIdx.x == 0) s_cb[NG] = meta[0];
      __syncthreads();
      if (threadIdx.x < 32) {
        // Warp 0: lane l takes a run of consecutive groups; exclusive prefix of
        // the heavy and light chunk counts over the runs.
        const int lane = threadIdx.x;
        const int per = (NG + 31) / 32;
        const int g0 = min(NG, lane * per), g1 = min(NG, g0 + per);
        int h = 0, l = 0;
        for (int g = g0; g < g1; ++g) {
          const int nc = s_cb[g + 1] - s_cb[g];
          if (counts[g] >= kHeavyRows) h += nc; else l += nc;
        }
        int hi = h, li = l;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int ho = __shfl_up_sync(0xffffffffu, hi, off);
          const int lo = __shfl_up_sync(0xffffffffu, li, off);
          if (lane >= off) {
            hi += ho;
            li += lo;
          }
        }
        int hrun = hi - h, lrun = li - l;
        for (int g = g0; g < g1; ++g) {
          const int nc = s_cb[g + 1] - s_cb[g];
          s_hcb[g] = hrun;
          s_lcb[g] = lrun;
          if (counts[g] >= kHeavyRows) hrun += nc; else lrun += nc;
        }
        if (lane == 31) {
          s_hcb[NG] = hi;
          s_lcb[NG] = li;
        }
      }
      __syncthreads();
      fill_tiles(tiles_up, Fu, NG, s_cb, s_hcb, s_lcb, err);
      fill_tiles(tiles_dn, Fd, NG, s_cb, s_hcb, s_lcb, err);
    }
  }
  const int c = blockIdx.x;
  const int t0 = c * kPermChunk;
  const int nt = min(kPermChunk, T_ - t0);
  for (int e = threadIdx.x; e < E; e += blockDim.x) mask[e] = 0u;
  __syncthreads();
  const int nent = nt * k;
  for (int q = threadIdx.x; q < nent; q += blockDim.x) {
    const int tl = q / k;
    const int e = idx[(int64_t)t0 * k + q];
    if (in_range(e, 0, E, err, 111)) atomicOr(&mask[e], 1u << tl);
  }
  __syncthreads();
  // blockIdx.y: a column slice of the copies (few tokens: several CTAs share a
  // chunk's copy); slice 0 also writes the row maps and the scales.
  const bool lead = blockIdx.y == 0;
  for (int q = threadIdx.x; q < nent; q += blockDim.x) {
    const int tl = q / k;
    const int e = idx[(int64_t)t0 * k + q];
    // An expert computed elsewhere (or, checked build, an id out of range): no row here.
    if ((kChecked && (e < 0 || e >= E)) || tab.slot[e] < 0) {
      if (lead) row_of[(int64_t)t0 * k + q] = -1;
      srow[q] = -1;
      continue;
    }
    const int rank = __popc(mask[e] & ((1u << tl) - 1u));
    const int row = chunk_base[(int64_t)c * E + e] + rank;
    if (!in_range(row, 0, (int64_t)T_ * k, err, 112)) {
      if (lead) row_of[(int64_t)t0 * k + q] = -1;
      srow[q] = -1;
      continue;
    }
    if (lead) {
      row_of[(int64_t)t0 * k + q] = row;
      tok_of[row] = t0 + tl;
      row_weight[row] = w[(int64_t)t0 * k + q];
    }
    srow[q] = row;
  }
  if (kMode == kNoCopy) return;
  __syncthreads();
  // Copy each token's row of x (bf16), or of its E4M3 codes, to its k permuted
  // rows in 16-byte chunks.
  const int nchunk = kMode == kCopyF8 ? d / 16 : d / 8;
  const int per = (nchunk + gridDim.y - 1) / gridDim.y;
  const int q0 = blockIdx.y * per, q1 = min(nchunk, q0 + per);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int tl = warp; tl < nt; tl += blockDim.x / 32) {
    const uint4* src = x + (int64_t)(t0 + tl) * nchunk;
    // Four 16-byte loads in flight per lane, then their copies.
    for (int q = q0 + lane; q < q1; q += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (q + 32 * u < q1) v[u] = src[q + 32 * u];
      for (int j = 0; j < k; ++j) {
        const int row = srow[tl * k + j];
        if (row < 0) continue;
        uint4* dst = xperm + (int64_t)row * nchunk;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (q + 32 * u < q1) dst[q + 32 * u] = v[u];
      }
    }
  }
  if (kMode != kCopyF8 || !lead) return;
  // MXFP8: each routed row's and each shared-expert row's scale bytes into its
  // GEMM chunk's scale blocks (4 K blocks per 32-bit word).
  const int nslab = d / 128;
  const int nent_all = nt * (k + S);
  for (int q = warp; q < nent_all; q += blockDim.x / 32) {
    const int tl = q / (k + S), j = q % (k + S);
    int g, rel;
    if (j < k) {
      g = idx[(int64_t)(t0 + tl) * k + j];
      if (srow[tl * k + j] < 0) continue;
      rel = srow[tl * k + j] - offsets[g];
    } else {
      if (t0 + tl < sb || t0 + tl >= se) continue;
      g = E + (j - k);
      rel = t0 + tl - sb;
    }
    const int64_t chunk = gchunk0[g] + rel / chunk_rows;
    if (!in_range(rel, 0, INT32_MAX, err, 113) || !in_range(chunk, 0, max_chunks, err, 114))
      continue;
    const int m = rel % chunk_rows;
    const uint32_t* srcs = reinterpret_cast<const uint32_t*>(xs + (int64_t)(t0 + tl) * (d / 32));
    for (int s4 = lane; s4 < nslab; s4 += 32)
      *reinterpret_cast<uint32_t*>(tok_sf + chunk_scale_offset(chunk, nslab, m, 4 * s4)) =
          srcs[s4];
  }
}

}  // namespace

cudaError_t launch_permute(const Resolved& r, const SlotTable& tab, int64_t T, const Layout& L,
                           char* ws, const int32_t* idx, const float* w, const void* x,
                           cudaStream_t st) {
  auto I32 = [&](size_t off) { return reinterpret_cast<int32_t*>(ws + off); };
  const int Fu = (r.I + 127) / 128, Fd = (r.d + 255) / 256;   // feature tiles per chunk
  (void)launch_pdl(permute_scan_kernel, dim3(1), dim3(kScanThreads), 0, st, r.E, r.S, (int)T, r.k,
                   (int)L.nperm, Fu, Fd, r.chunk_rows, tab,
                   r.n_local, r.sb, r.se, I32(L.chunk_counts), I32(L.chunk_base), I32(L.counts),
                   I32(L.offsets), reinterpret_cast<Chunk*>(ws + L.chunks), I32(L.meta),
                   I32(L.gchunk0), (int)L.max_chunks, I32(L.err));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // Few chunks (a decode step): split each chunk's row copies over column
  // slices so that about two CTAs per SM copy.
  const int64_t target = 2 * (r.num_sms > 0 ? r.num_sms : 148);
  const int64_t want = (target + L.nperm - 1) / L.nperm;
  const int slices = r.act_bf16 ? (int)std::max<int64_t>(1, std::min<int64_t>(16, want)) : 1;
  const dim3 grid((unsigned)L.nperm, (unsigned)slices);
  float* rw = reinterpret_cast<float*>(ws + L.row_weight);
  const int32_t* base = I32(L.chunk_base);
  if (r.fp8)
    (void)launch_pdl(permute_scatter_kernel<kCopyF8>, grid, dim3(kScatterThreads), 0, st, r.E, r.S, (int)T,
                     r.k, r.d, r.chunk_rows, tab, r.sb, r.se, idx, w, base, I32(L.offsets),
                     I32(L.gchunk0), I32(L.row_of), I32(L.tok_of), rw,
                     reinterpret_cast<const uint4*>(ws + L.xq),
                     reinterpret_cast<uint4*>(ws + L.xperm),
                     reinterpret_cast<const uint8_t*>(ws + L.xs),
                     reinterpret_cast<uint8_t*>(ws + L.tok_sf), (int)L.max_chunks, I32(L.counts), I32(L.meta), Fu, Fd,
                     reinterpret_cast<int2*>(ws + L.tiles_up),
                     reinterpret_cast<int2*>(ws + L.tiles_down), I32(L.err));
  else if (r.dtype == KT_DTYPE_BF16)
    (void)launch_pdl(permute_scatter_kernel<kCopyBf16>, grid, dim3(kScatterThreads), 0, st, r.E, r.S, (int)T,
                     r.k, r.d, r.chunk_rows, tab, r.sb, r.se, idx, w, base, I32(L.offsets),
                     I32(L.gchunk0), I32(L.row_of), I32(L.tok_of), rw,
                     reinterpret_cast<const uint4*>(x), reinterpret_cast<uint4*>(ws + L.xperm),
                     nullptr, nullptr, (int)L.max_chunks, I32(L.counts), I32(L.meta), Fu, Fd,
                     reinterpret_cast<int2*>(ws + L.tiles_up),
                     reinterpret_cast<int2*>(ws + L.tiles_down), I32(L.err));
  else
    (void)launch_pdl(permute_scatter_kernel<kNoCopy>, grid, dim3(kScatterThreads), 0, st, r.E, r.S, (int)T,
                     r.k, r.d, r.chunk_rows, tab, r.sb, r.se, idx, w, base, I32(L.offsets),
                     I32(L.gchunk0), I32(L.row_of), I32(L.tok_of), rw, nullptr, nullptr, nullptr,
                     nullptr, (int)L.max_chunks, I32(L.counts), I32(L.meta), Fu, Fd,
                     reinterpret_cast<int2*>(ws + L.tiles_up),
                     reinterpret_cast<int2*>(ws + L.tiles_down), I32(L.err));
  return cudaGetLastError();
}

}  // namespace ktmoe
