// merge.cu -- the online-softmax merge of partial attention results (the requester's side
// of the Route primitive) and the result of a partial attention over an empty shard.
//
// Operation (page "Move the Query, Not the Cache: Characterizing Cross-Instance Latent
// Attention Redistribution Across GPU Fabrics", explainer "Technisches Resuemee: Den Query
// bewegen, nicht den Cache" -> "Methodik" -> "Primitiv-Vergleich": the owner of a KV shard
// computes the partial attention of the routed queries and the requester merges the small
// results with an online softmax).  For each query row and parts t = 0 .. n-1 with partial
// outputs O_t (normalised over the part's keys) and log-sum-exps lse_t:
//     M = max_t lse_t,  w_t = exp(lse_t - M),  O = sum_t w_t O_t / sum_t w_t,
//     lse = M + log(sum_t w_t);
// a row whose parts are all empty (lse_t = -inf) gives O = 0 and lse = -inf.
//
// The merge reads n * (4 D + 4) bytes and writes 2 D (+ 4) bytes per row and does a few
// flops per byte: it is bound by HBM bandwidth.  One thread handles four consecutive fp32
// columns of one row (16-byte loads; consecutive threads cover consecutive columns, then
// rows), so every warp-wide load is a contiguous 512-byte span of one part.  The grid covers
// the whole merge in one pass (one chunk per thread; the block scheduler fills the SMs as
// blocks finish), and the partial outputs, read exactly once, are loaded without allocating
// in L1: against a grid of 8 resident blocks per SM striding over the rows, 76 MB merge in
// 16.4 instead of 18.5 us and 305-485 MB at 6.5-7.2 instead of 5.5-6.2 TB/s.  The part count
// is a template bound (2, 4, 8 or 16) so that all of a thread's loads are in flight together.
#include "xs_internal.cuh"

namespace xs {
namespace {

// 16-byte global load that does not allocate in L1 (each partial output is read once).
__device__ __forceinline__ float4 ld_stream_f4(const float *ptr) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(ptr));
  return v;
}

// MAXN >= p.n: the loads of every part's lse and O chunk are issued before any is used, so
// each thread has 2n loads in flight.
template <int MAXN>
__global__ void __launch_bounds__(256) lse_merge_kernel(const __grid_constant__ MergeParams p) {
  const int nq = p.D >> 2;  // float4 chunks per row
  const long long total = p.rows * nq;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; g < total; g += stride) {
    const long long r = g / nq;
    const int c = static_cast<int>(g - r * nq);
    float lv[MAXN];
    float4 xv[MAXN];
#pragma unroll
    for (int t = 0; t < MAXN; ++t) {
      if (t < p.n) {
        lv[t] = __ldg(p.lse[t] + r);
        xv[t] = ld_stream_f4(p.o[t] + r * p.D + 4 * c);
      } else {
        lv[t] = -INFINITY;
        xv[t] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int t = 0; t < MAXN; ++t) M = fmaxf(M, lv[t]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float W = 0.f;
    if (M > -INFINITY) {
#pragma unroll
      for (int t = 0; t < MAXN; ++t) {
        const float w = expf(lv[t] - M);  // exp(-inf) = 0 for an empty part
        W += w;
        // An empty part contributes nothing, whatever its O holds.
        acc.x += w > 0.f ? w * xv[t].x : 0.f;
        acc.y += w > 0.f ? w * xv[t].y : 0.f;
        acc.z += w > 0.f ? w * xv[t].z : 0.f;
        acc.w += w > 0.f ? w * xv[t].w : 0.f;
      }
    }
    const float inv = M > -INFINITY ? 1.f / W : 0.f;
    uint2 packed;
    packed.x = ptx::pack_bf16(acc.x * inv, acc.y * inv);
    packed.y = ptx::pack_bf16(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.out) + (r * p.D + 4 * c) * 2)[0] = packed;
    if (c == 0 && p.lse_out != nullptr) p.lse_out[r] = M > -INFINITY ? M + logf(W) : -INFINITY;
  }
}

__global__ void __launch_bounds__(256) partial_empty_kernel(float *o, float *lse, long long rows, int D) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long n4 = rows * (D >> 2);
  for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; g < n4; g += stride)
    reinterpret_cast<float4 *>(o)[g] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; g < rows; g += stride)
    lse[g] = -INFINITY;
}

int grid_for(long long work, int threads) {
  const int sms = device_sm_count();
  if (sms <= 0) return -1;
  const long long blocks = (work + threads - 1) / threads;
  const long long cap = static_cast<long long>(sms) * 8;  // 8 resident blocks of 256 per SM
  return static_cast<int>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace

cudaError_t launch_lse_merge(const MergeParams &p, cudaStream_t stream) {
  // One pass over all chunks; beyond 2^22 blocks (2^30 chunks) the kernel's grid-stride loop
  // takes the rest.
  const long long blocks = (p.rows * (p.D >> 2) + 255) / 256;
  const int grid = static_cast<int>(blocks < (1ll << 22) ? (blocks > 0 ? blocks : 1) : (1ll << 22));
  if (p.n <= 2) lse_merge_kernel<2><<<grid, 256, 0, stream>>>(p);
  else if (p.n <= 4) lse_merge_kernel<4><<<grid, 256, 0, stream>>>(p);
  else if (p.n <= 8) lse_merge_kernel<8><<<grid, 256, 0, stream>>>(p);
  else lse_merge_kernel<16><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_partial_empty(float *o, float *lse, long long rows, int D, cudaStream_t stream) {
  const int grid = grid_for(rows * (D >> 2), 256);
  if (grid <= 0) return cudaErrorInvalidDevice;
  partial_empty_kernel<<<grid, 256, 0, stream>>>(o, lse, rows, D);
  return cudaGetLastError();
}

}  // namespace xs
