// exchange.cu -- the stand-alone post-attention All-to-All (serial baseline), the Burst-Gap
// store microbenchmark and the bounded-wait self-test.
#include "xs_internal.cuh"

namespace xs {
namespace {

// ---------------------------------------------------------------- re-layout
// dest[r][b, s_local, h, :] = src[b, h, r*S_local + s_local, :]
// One warp per destination row (r, b, s_local): that row is H*D contiguous words in dest,
// read as H runs of D contiguous words from src.  16-byte loads and stores, four in flight
// per lane.  HBM-bound: 2 * B*H*S*D*2 bytes moved.
__global__ void __launch_bounds__(256) relayout_kernel(const __grid_constant__ RelayoutParams p) {
  const int nch = p.D >> 3;              // 16-byte chunks per (h) run
  const int row_chunks = p.H * nch;      // 16-byte chunks per destination row
  const long long rows_per_rank = static_cast<long long>(p.B) * p.S_local;
  const long long n_rows = rows_per_rank * p.P;
  const int lane = threadIdx.x & 31;
  const long long warp0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const uint4 *src = static_cast<const uint4 *>(p.src);
  const long long head_stride = static_cast<long long>(p.S) * nch;  // chunks between heads

  for (long long row = warp0; row < n_rows; row += n_warps) {
    const int r = static_cast<int>(row / rows_per_rank);
    const long long rem = row - r * rows_per_rank;
    const int b = static_cast<int>(rem / p.S_local);
    const int sl = static_cast<int>(rem - static_cast<long long>(b) * p.S_local);
    const int s = r * p.S_local + sl;
    uint4 *d = static_cast<uint4 *>(p.dest[r]) + rem * row_chunks;
    const uint4 *sb = src + (static_cast<long long>(b) * p.H * p.S + s) * nch;
    int i = lane;
    for (; i + 96 < row_chunks; i += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int ii = i + 32 * u;
        const int h = ii / nch;
        v[u] = __ldg(sb + h * head_stride + (ii - h * nch));
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) d[i + 32 * u] = v[u];
    }
    for (; i < row_chunks; i += 32) {
      const int h = i / nch;
      d[i] = __ldg(sb + h * head_stride + (i - h * nch));
    }
  }
}

// ---------------------------------------------------------------- pre-attention exchange
// dst[b, h, r*S_local + s_local, :] = src[r][b, s_local, head_offset + h, :], h < H_local.
// One warp per source row (r, b, s_local): H_local*D contiguous words of src[r], written as
// H_local runs of D words into the head-major dst.  16-byte loads and stores, four in flight.
__global__ void __launch_bounds__(256) pre_relayout_kernel(const __grid_constant__ PreRelayoutParams p) {
  const int nch = p.D >> 3;
  const int row_chunks = p.H_local * nch;
  const long long rows_per_rank = static_cast<long long>(p.B) * p.S_local;
  const long long n_rows = rows_per_rank * p.P;
  const int lane = threadIdx.x & 31;
  const long long warp0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  uint4 *dst = static_cast<uint4 *>(p.dst);
  const long long head_stride = static_cast<long long>(p.S) * nch;  // chunks between heads of dst
  for (long long row = warp0; row < n_rows; row += n_warps) {
    const int r = static_cast<int>(row / rows_per_rank);
    const long long rem = row - r * rows_per_rank;
    const int b = static_cast<int>(rem / p.S_local);
    const int sl = static_cast<int>(rem - static_cast<long long>(b) * p.S_local);
    const int s = r * p.S_local + sl;
    const uint4 *src = static_cast<const uint4 *>(p.src[r]) +
                       (rem * p.H_total + p.head_offset) * nch;
    uint4 *db = dst + (static_cast<long long>(b) * p.H_local * p.S + s) * nch;
    int i = lane;
    for (; i + 96 < row_chunks; i += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = __ldg(src + i + 32 * u);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int ii = i + 32 * u;
        const int h = ii / nch;
        db[h * head_stride + (ii - h * nch)] = v[u];
      }
    }
    for (; i < row_chunks; i += 32) {
      const int h = i / nch;
      db[h * head_stride + (i - h * nch)] = __ldg(src + i);
    }
  }
}

// ---------------------------------------------------------------- Burst-Gap probe
// Each CTA is one producer.  Per burst: stamp, every thread issues its part of the
// producer's share of 16-byte stores, the CTA syncs (all stores issued, none waited for),
// stamp, then each thread runs a dependent FMA chain (the compute gap), stamp.
__global__ void burst_probe_kernel(const __grid_constant__ BurstParams p) {
  __shared__ unsigned long long t_start, t_issued, g_start;
  const int pid = blockIdx.x;
  float acc = static_cast<float>(threadIdx.x) * 1e-3f;
  for (int i = 0; i < p.n_bursts; ++i) {
    __syncthreads();
    if (threadIdx.x == 0) {
      g_start = ptx::globaltimer();
      t_start = clock64();
    }
    __syncthreads();
    const long long first =
        ((static_cast<long long>(i) * p.producers + pid) * p.share_chunks) % p.scratch_chunks;
    for (long long c = threadIdx.x; c < p.share_chunks; c += blockDim.x) {
      long long idx = first + c;
      if (idx >= p.scratch_chunks) idx -= p.scratch_chunks;
      ptx::st_global_v4(p.scratch + idx,
                        make_uint4(static_cast<uint32_t>(i), static_cast<uint32_t>(pid),
                                   static_cast<uint32_t>(c), 0x5a5a5a5au));
    }
    __syncthreads();
    if (threadIdx.x == 0) t_issued = clock64();
    for (long long g = 0; g < p.gap_iters; ++g) acc = fmaf(acc, 0.999999f, 1e-6f);
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long *st = p.stamps + (static_cast<long long>(pid) * p.n_bursts + i) * 4;
      st[0] = t_start;
      st[1] = t_issued;
      st[2] = clock64();
      st[3] = g_start;
    }
  }
  // Keep the FMA chain observable (never true for the values above).
  if (acc == -1.0f) p.scratch[0] = make_uint4(0, 0, 0, 0);
}

// ---------------------------------------------------------------- bounded-wait self-test
__global__ void wait_selftest_kernel(int *status, long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_u32(&bar), 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl ctl{&abort_flag, status, limit_ns};
    // Nothing ever arrives on `bar`: the wait must give up and report a timeout.
    bounded_wait(ptx::smem_u32(&bar), 0, ctl);
  }
}

// ---------------------------------------------------------------- slab arrival wait
// One thread polls the counter with system-scope acquire loads, sleeping between polls, until
// it reaches target or the limit passes (then XS_ERR_TIMEOUT is recorded).  Stream order makes
// the kernels enqueued after this one see every store the counted releases covered.
__global__ void slab_wait_kernel(const unsigned int *flag, unsigned int target, long long limit_ns,
                                 int *status) {
  const uint64_t t0 = ptx::globaltimer();
  while (static_cast<int>(ptx::ld_acquire_sys(flag) - target) < 0) {
    if (static_cast<long long>(ptx::globaltimer() - t0) > limit_ns) {
      atomicCAS(status, kStatusOk, kStatusTimeout);
      return;
    }
    __nanosleep(1000);
  }
}

}  // namespace

cudaError_t launch_slab_wait(const unsigned int *flag, unsigned int target, long long limit_ns,
                             int *status, cudaStream_t stream) {
  slab_wait_kernel<<<1, 1, 0, stream>>>(flag, target, limit_ns, status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- fixed probe scratch
// Scratch of the allocation-free probe entry point: a fixed array in the module's global
// memory, reserved on every device that loads the library until the process exits.  Host
// code must not pass `g_probe_scratch` itself to a kernel (on the host it names a host-side
// stand-in); it passes the device address that cudaGetSymbolAddress returns.
static __device__ __align__(256) uint4 g_probe_scratch[kStaticProbeScratchBytes / 16];

cudaError_t static_probe_scratch(uint4 **out) {
  // Looked up on every call, in the context current on the calling thread: the address
  // belongs to the module loaded in that context, so a cached value would be wrong for a
  // caller that switches contexts (cuCtxSetCurrent) or after cudaDeviceReset.  The lookup
  // allocates nothing; the first one in a context may load the module, so the first call
  // should precede any stream capture.
  void *p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_probe_scratch);
  if (e != cudaSuccess) return e;
  *out = static_cast<uint4 *>(p);
  return cudaSuccess;
}

cudaError_t launch_relayout(const RelayoutParams &p, cudaStream_t stream) {
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const long long n_rows = static_cast<long long>(p.B) * p.S_local * p.P;
  const long long warps_needed = n_rows;
  long long blocks = (warps_needed + 7) / 8;
  const long long cap = static_cast<long long>(sms) * 8;  // 8 resident 256-thread CTAs per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  relayout_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_pre_relayout(const PreRelayoutParams &p, cudaStream_t stream) {
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const long long n_rows = static_cast<long long>(p.B) * p.S_local * p.P;
  long long blocks = (n_rows + 7) / 8;
  const long long cap = static_cast<long long>(sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  pre_relayout_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_burst_probe(const BurstParams &p, int threads, cudaStream_t stream) {
  burst_probe_kernel<<<p.producers, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int *status, long long limit_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace xs
