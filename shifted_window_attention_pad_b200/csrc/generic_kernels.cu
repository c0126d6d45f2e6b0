// generic_kernels.cu -- portable per-token CUDA kernels for shifted-window attention.
//
// One thread per query (forward, backward rows) or per key (backward columns),
// fp32 arithmetic, any window / shift / head size the ABI accepts, fp32 or bf16
// storage. These carry the fp32 path and every shape the tcgen05 kernels do not
// take. Steps (TERRA page, Abstract "shifted-window execution" of a window-based
// Swin Transformer; Table I padded resolution): pad, cyclic shift and window
// partition are address arithmetic (geometry.cuh); each window runs masked
// softmax attention with the relative-position bias; results go straight back
// to the grid positions they came from.
#include <cuda_bf16.h>
#include <math.h>

#include "kernels.h"

namespace swin {

namespace {

constexpr int kMaxHd = 256;
constexpr int kThreads = 128;

__device__ __forceinline__ float ld(const float* p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st(float* p, float x) { *p = x; }
__device__ __forceinline__ void st(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Per-window slot table staged in shared memory: element offset of the token's
// row for head h (or -1 for a slot outside the stored grid), region label (a
// distinct negative value -1 - slot for a token beyond the valid extent, so it
// pairs with nothing), slot coordinates.
struct SlotTab {
  long long* off;
  int* label;
  int* iy;
  int* ix;
};

__device__ SlotTab stage_slots(const Geo& g, long long win, int h, unsigned char* smem) {
  SlotTab t;
  t.off = reinterpret_cast<long long*>(smem);
  t.label = reinterpret_cast<int*>(t.off + g.N);
  t.iy = t.label + g.N;
  t.ix = t.iy + g.N;
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) {
    const SlotInfo s = slot_info(g, win, i);
    t.off[i] = s.stored ? (token_of(g, s) * g.heads + h) * g.hd : -1;
    t.label[i] = s.valid ? s.label : -1 - i;
    t.iy[i] = s.iy;
    t.ix[i] = s.ix;
  }
  __syncthreads();
  return t;
}

// Key j is allowed for query i: both real tokens in the same shift region.
__device__ __forceinline__ bool allowed(const SlotTab& t, int i, int j) {
  return t.label[i] >= 0 && t.label[i] == t.label[j];
}

__host__ size_t slot_smem(const Geo& g) { return (size_t)g.N * (sizeof(long long) + 3 * sizeof(int)); }

template <typename T>
__device__ float dot(const T* a, const T* b, int n) {
  float acc = 0.f;
  for (int e = 0; e < n; ++e) acc = fmaf(ld(a + e), ld(b + e), acc);
  return acc;
}

__global__ void index_map_kernel(Geo g, int32_t* map) {
  const long long total = g.n_win * g.N;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const long long win = t / g.N;
    const SlotInfo s = slot_info(g, win, (int)(t - win * g.N));
    map[t] = s.valid ? (int32_t)token_of(g, s) : -1;
  }
}

// Forward: block = (window, head); thread = query slot.
template <typename T>
__global__ void generic_fwd_kernel(Geo g, const T* __restrict__ q, const T* __restrict__ k,
                                   const T* __restrict__ v, const float* __restrict__ table,
                                   T* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(16) unsigned char smem[];
  const long long win = blockIdx.x;
  const int h = blockIdx.y;
  const SlotTab t = stage_slots(g, win, h, smem);
  const float scale = 1.0f / sqrtf((float)g.hd);
  float acc[kMaxHd];
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) {
    if (t.off[i] < 0) continue;
    if (t.label[i] < 0) {   // stored token beyond the valid extent: zeros
      for (int e = 0; e < g.hd; ++e) st(out + t.off[i] + e, 0.f);
      if (lse) lse[t.off[i] / g.hd] = 0.f;
      continue;
    }
    const T* qi = q + t.off[i];
    float m = -INFINITY;
    for (int j = 0; j < g.N; ++j) {
      if (!allowed(t, i, j)) continue;
      const float a = scale * dot(qi, k + t.off[j], g.hd) +
                      table[rel_index(g, t.iy[i], t.ix[i], t.iy[j], t.ix[j]) * g.heads + h];
      m = fmaxf(m, a);
    }
    for (int e = 0; e < g.hd; ++e) acc[e] = 0.f;
    float l = 0.f;
    for (int j = 0; j < g.N; ++j) {
      if (!allowed(t, i, j)) continue;
      const float a = scale * dot(qi, k + t.off[j], g.hd) +
                      table[rel_index(g, t.iy[i], t.ix[i], t.iy[j], t.ix[j]) * g.heads + h];
      const float p = expf(a - m);
      l += p;
      const T* vj = v + t.off[j];
      for (int e = 0; e < g.hd; ++e) acc[e] = fmaf(p, ld(vj + e), acc[e]);
    }
    const float inv = 1.0f / l;
    for (int e = 0; e < g.hd; ++e) st(out + t.off[i] + e, acc[e] * inv);
    if (lse) lse[t.off[i] / g.hd] = m + logf(l);
  }
}

// Recomputes the softmax statistics of query row i: max m and sum l.
template <typename T>
__device__ void row_stats(const Geo& g, const SlotTab& t, int i, int h, const T* q, const T* k,
                          const float* table, float scale, float& m, float& l) {
  const T* qi = q + t.off[i];
  m = -INFINITY;
  for (int j = 0; j < g.N; ++j) {
    if (!allowed(t, i, j)) continue;
    m = fmaxf(m, scale * dot(qi, k + t.off[j], g.hd) +
                     table[rel_index(g, t.iy[i], t.ix[i], t.iy[j], t.ix[j]) * g.heads + h]);
  }
  l = 0.f;
  for (int j = 0; j < g.N; ++j) {
    if (!allowed(t, i, j)) continue;
    l += expf(scale * dot(qi, k + t.off[j], g.hd) +
              table[rel_index(g, t.iy[i], t.ix[i], t.iy[j], t.ix[j]) * g.heads + h] - m);
  }
}

// Backward rows: block = (window, head); thread = query i. Stores (m, l, D) per
// query and dq_i = scale * sum_j dS_ij k_j.
template <typename T>
__global__ void generic_bwd_rows_kernel(Geo g, const T* __restrict__ q, const T* __restrict__ k,
                                        const T* __restrict__ v, const float* __restrict__ table,
                                        const T* __restrict__ dout, T* __restrict__ dq,
                                        float* __restrict__ stats) {
  extern __shared__ __align__(16) unsigned char smem[];
  const long long win = blockIdx.x;
  const int h = blockIdx.y;
  const SlotTab t = stage_slots(g, win, h, smem);
  const float scale = 1.0f / sqrtf((float)g.hd);
  float acc[kMaxHd];
  for (int i = threadIdx.x; i < g.N; i += blockDim.x) {
    float* st3 = stats + ((win * g.heads + h) * g.N + i) * 3;
    if (t.off[i] < 0 || t.label[i] < 0) {
      st3[0] = 0.f; st3[1] = 1.f; st3[2] = 0.f;
      if (t.off[i] >= 0)
        for (int e = 0; e < g.hd; ++e) st(dq + t.off[i] + e, 0.f);
      continue;
    }
    float m, l;
    row_stats(g, t, i, h, q, k, table, scale, m, l);
    const T* qi = q + t.off[i];
    const T* doi = dout + t.off[i];
    float D = 0.f;
    for (int j = 0; j < g.N; ++j) {
      if (!allowed(t, i, j)) continue;
      const float p = expf(scale * dot(qi, k + t.off[j], g.hd) +
                           table[rel_index(g, t.iy[i], t.ix[i], t.iy[j], t.ix[j]) * g.heads + h] -
                           m) / l;
      D = fmaf(p, dot(doi, v + t.off[j], g.hd), D);
    }
    for (int e = 0; e < g.hd; ++e) acc[e] = 0.f;
    for (int j = 0; j < g.N; ++j) {
      if (!allowed(t, i, j)) continue;
      const float p = expf(scale * dot(qi, k + t.off[j], g.hd) +
                           table[rel_index(g, t.iy[i], t.ix[i], t.iy[j], t.ix[j]) * g.heads + h] -
                           m) / l;
      const float ds = p * (dot(doi, v + t.off[j], g.hd) - D);
      const T* kj = k + t.off[j];
      for (int e = 0; e < g.hd; ++e) acc[e] = fmaf(ds, ld(kj + e), acc[e]);
    }
    for (int e = 0; e < g.hd; ++e) st(dq + t.off[i] + e, scale * acc[e]);
    st3[0] = m; st3[1] = l; st3[2] = D;
  }
}

// Backward columns: block = (window, head); thread = key j. dk_j and dv_j.
template <typename T>
__global__ void generic_bwd_cols_kernel(Geo g, const T* __restrict__ q, const T* __restrict__ k,
                                        const T* __restrict__ v, const float* __restrict__ table,
                                        const T* __restrict__ dout, T* __restrict__ dk,
                                        T* __restrict__ dv, const float* __restrict__ stats) {
  extern __shared__ __align__(16) unsigned char smem[];
  const long long win = blockIdx.x;
  const int h = blockIdx.y;
  const SlotTab t = stage_slots(g, win, h, smem);
  const float scale = 1.0f / sqrtf((float)g.hd);
  float ak[kMaxHd], av[kMaxHd];
  for (int j = threadIdx.x; j < g.N; j += blockDim.x) {
    if (t.off[j] < 0) continue;
    for (int e = 0; e < g.hd; ++e) ak[e] = av[e] = 0.f;
    if (t.label[j] < 0) {   // stored token beyond the valid extent: zeros
      for (int e = 0; e < g.hd; ++e) {
        st(dk + t.off[j] + e, 0.f);
        st(dv + t.off[j] + e, 0.f);
      }
      continue;
    }
    const T* kj = k + t.off[j];
    const T* vj = v + t.off[j];
    for (int i = 0; i < g.N; ++i) {
      if (!allowed(t, j, i)) continue;
      const float* st3 = stats + ((win * g.heads + h) * g.N + i) * 3;
      const T* qi = q + t.off[i];
      const T* doi = dout + t.off[i];
      const float p = expf(scale * dot(qi, kj, g.hd) +
                           table[rel_index(g, t.iy[i], t.ix[i], t.iy[j], t.ix[j]) * g.heads + h] -
                           st3[0]) / st3[1];
      const float ds = p * (dot(doi, vj, g.hd) - st3[2]);
      for (int e = 0; e < g.hd; ++e) {
        ak[e] = fmaf(ds, ld(qi + e), ak[e]);
        av[e] = fmaf(p, ld(doi + e), av[e]);
      }
    }
    for (int e = 0; e < g.hd; ++e) {
      st(dk + t.off[j] + e, scale * ak[e]);
      st(dv + t.off[j] + e, av[e]);
    }
  }
}

// Bias-gradient partial of one (window, head): thread = table entry (dy, dx);
// sums dS_ij over the pairs with that offset, queries in slot order.
template <typename T>
__global__ void generic_dbias_partial_kernel(Geo g, const T* __restrict__ q,
                                             const T* __restrict__ k, const T* __restrict__ v,
                                             const float* __restrict__ table,
                                             const T* __restrict__ dout,
                                             const float* __restrict__ stats, int bins_pad,
                                             float* __restrict__ partial) {
  extern __shared__ __align__(16) unsigned char smem[];
  const long long win = blockIdx.x;
  const int h = blockIdx.y;
  const SlotTab t = stage_slots(g, win, h, smem);
  const float scale = 1.0f / sqrtf((float)g.hd);
  for (int bin = threadIdx.x; bin < bins_pad; bin += blockDim.x) {
    float sum = 0.f;
    if (bin < g.bins) {
      const int dy = bin / (2 * g.ww - 1) - (g.wh - 1);
      const int dx = bin % (2 * g.ww - 1) - (g.ww - 1);
      for (int i = 0; i < g.N; ++i) {
        const int jy = t.iy[i] - dy, jx = t.ix[i] - dx;
        if (jy < 0 || jy >= g.wh || jx < 0 || jx >= g.ww) continue;
        const int j = jy * g.ww + jx;
        if (!allowed(t, i, j)) continue;
        const float* st3 = stats + ((win * g.heads + h) * g.N + i) * 3;
        const float p = expf(scale * dot(q + t.off[i], k + t.off[j], g.hd) + table[bin * g.heads + h] -
                             st3[0]) / st3[1];
        sum += p * (dot(dout + t.off[i], v + t.off[j], g.hd) - st3[2]);
      }
    }
    partial[(win * g.heads + h) * bins_pad + bin] = sum;
  }
}

// dtable[bin][h] = sum over units u of partial[u][h][bin], in a fixed order: a
// block owns one head and 32 table entries; its 8 lanes per entry each sum
// every 8th unit in increasing order, then the 8 lane sums are added in lane
// order. The result does not depend on timing, so it is bitwise repeatable.
__global__ void dbias_reduce_kernel(int heads, int bins, int bins_pad, long long n_units,
                                    const float* __restrict__ partial, float* __restrict__ dtable) {
  __shared__ float lane_sum[8][33];
  const int h = blockIdx.y;
  const int bl = threadIdx.x & 31, ul = threadIdx.x >> 5;
  const int bin = blockIdx.x * 32 + bl;
  float s = 0.f;
  if (bin < bins)
    for (long long u = ul; u < n_units; u += 8) s += partial[(u * heads + h) * bins_pad + bin];
  lane_sum[ul][bl] = s;
  __syncthreads();
  if (ul == 0 && bin < bins) {
    float tot = 0.f;
    for (int i = 0; i < 8; ++i) tot += lane_sum[i][bl];
    dtable[bin * heads + h] = tot;
  }
}

template <typename T>
cudaError_t fwd_impl(const Geo& g, const void* q, const void* k, const void* v,
                     const float* table, void* out, float* lse, cudaStream_t st) {
  const dim3 grid((unsigned)g.n_win, g.heads);
  generic_fwd_kernel<T><<<grid, kThreads, slot_smem(g), st>>>(
      g, (const T*)q, (const T*)k, (const T*)v, table, (T*)out, lse);
  note_launch();
  return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_impl(const Geo& g, const void* q, const void* k, const void* v,
                     const float* table, const void* dout, void* dq, void* dk, void* dv,
                     float* dtable, void* ws, cudaStream_t st) {
  char* base = (char*)ws + kWsHeader;
  float* stats = (float*)base;
  const int bp = bins_padded(g.bins);
  float* partial = (float*)(base + align256((size_t)g.n_win * g.heads * g.N * 3 * sizeof(float)));
  const dim3 grid((unsigned)g.n_win, g.heads);
  const size_t sm = slot_smem(g);
  generic_bwd_rows_kernel<T><<<grid, kThreads, sm, st>>>(g, (const T*)q, (const T*)k,
                                                         (const T*)v, table, (const T*)dout,
                                                         (T*)dq, stats);
  generic_bwd_cols_kernel<T><<<grid, kThreads, sm, st>>>(g, (const T*)q, (const T*)k,
                                                         (const T*)v, table, (const T*)dout,
                                                         (T*)dk, (T*)dv, stats);
  generic_dbias_partial_kernel<T><<<grid, kThreads, sm, st>>>(
      g, (const T*)q, (const T*)k, (const T*)v, table, (const T*)dout, stats, bp, partial);
  note_launch(3);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return dbias_reduce(g, partial, g.n_win, dtable, st);
}

}  // namespace

size_t generic_workspace(const Geo& g) {
  return kWsHeader + align256((size_t)g.n_win * g.heads * g.N * 3 * sizeof(float)) +
         align256((size_t)g.n_win * g.heads * bins_padded(g.bins) * sizeof(float));
}

cudaError_t generic_forward(const Geo& g, int dtype, const void* q, const void* k, const void* v,
                            const float* table, void* out, float* lse, void*, cudaStream_t st) {
  return dtype == SWIN_DTYPE_F32 ? fwd_impl<float>(g, q, k, v, table, out, lse, st)
                                 : fwd_impl<__nv_bfloat16>(g, q, k, v, table, out, lse, st);
}

cudaError_t generic_backward(const Geo& g, int dtype, const void* q, const void* k,
                             const void* v, const float* table, const void* dout, void* dq,
                             void* dk, void* dv, float* dtable, void* ws, cudaStream_t st) {
  return dtype == SWIN_DTYPE_F32
             ? bwd_impl<float>(g, q, k, v, table, dout, dq, dk, dv, dtable, ws, st)
             : bwd_impl<__nv_bfloat16>(g, q, k, v, table, dout, dq, dk, dv, dtable, ws, st);
}

cudaError_t index_map(const Geo& g, int32_t* map, cudaStream_t st) {
  const long long total = g.n_win * g.N;
  const int blocks = (int)((total + 255) / 256 < 148 * 8 ? (total + 255) / 256 : 148 * 8);
  index_map_kernel<<<blocks > 0 ? blocks : 1, 256, 0, st>>>(g, map);
  note_launch();
  return cudaGetLastError();
}

cudaError_t dbias_reduce(const Geo& g, const float* partial, long long n_units, float* dtable,
                         cudaStream_t st) {
  const dim3 grid((g.bins + 31) / 32, g.heads);
  dbias_reduce_kernel<<<grid, 256, 0, st>>>(g.heads, g.bins, bins_padded(g.bins), n_units,
                                            partial, dtable);
  note_launch();
  return cudaGetLastError();
}

}  // namespace swin
