// xs_internal.cuh -- types shared by the kernels and the C-ABI layer of libxs.so.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "ptx.cuh"

namespace xs {

constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = 4;  // XS_ERR_TIMEOUT
constexpr int kMaxRanks = 16;

// Default bound of every on-device wait (global-timer nanoseconds).  A healthy wait in any
// kernel here lasts microseconds; two seconds only ever trips when something is wrong.
constexpr long long kWaitLimitNs = 2000000000LL;
// Bound of the waits a CTA runs while shutting down after an abort (for its own copies and
// MMAs in flight, which end within microseconds).  Kept apart from the caller-set wait limit,
// so that a short limit never lets a CTA exit before its own asynchronous work has landed.
constexpr long long kDrainLimitNs = 2000000000LL;

// Bounded wait on an mbarrier phase.  Returns false when the CTA-wide abort flag is set or
// the limit passes; in the latter case it raises the abort flag and records XS_ERR_TIMEOUT
// in *status (first error wins).  Never traps.
struct WaitCtl {
  volatile int *abort_flag;  // shared memory
  int *status;               // device, nullable
  long long limit_ns;
};

__device__ __forceinline__ void raise_timeout(const WaitCtl &c) {
  *c.abort_flag = 1;
  if (c.status) atomicCAS(c.status, kStatusOk, kStatusTimeout);
}

#ifndef XS_WAIT_SLEEP_NS
#define XS_WAIT_SLEEP_NS 20000
#endif

__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, const WaitCtl &c) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (true) {
    if (ptx::mbar_try_wait_sleep(bar, parity, XS_WAIT_SLEEP_NS)) return true;
    if (*c.abort_flag) return false;
    if (static_cast<long long>(ptx::globaltimer() - t0) > c.limit_ns) {
      raise_timeout(c);
      return false;
    }
  }
}

// Wait used only while shutting down after an abort: ignores the abort flag, still bounded.
__device__ __forceinline__ bool bounded_wait_drain(uint32_t bar, uint32_t parity, long long limit_ns) {
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (static_cast<long long>(ptx::globaltimer() - t0) > limit_ns) return false;
  }
  return true;
}

// ---------------------------------------------------------------- attention
enum EpilogueKind : int {
  kHeadMajor = 0,   // out[b, h, s, :]
  kSeqScatter = 1,  // dest[r][b, s_local, h, :]  (fused post-attention All-to-All)
  kPartial = 2,     // out[b, h, s, :] in fp32 plus lse[b, h, s] (partial attention of a shard)
  kSeqScatterSpans = 3,  // kSeqScatter, recording each tile's store-issue span in spans[]
};

struct AttnParams {
  CUtensorMap tm_q;  // 3-D view {D, S, B*H} of q, box {64, 128, 1}, 128-byte swizzle
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  void *out;               // kHeadMajor (bf16), kPartial (fp32)
  float *lse;              // kPartial: natural-log log-sum-exp of each query row
  unsigned long long *spans;  // kSeqScatterSpans: [n_items][2 tiles][4 warps][3]
  void *dest[kMaxRanks];   // kSeqScatter
  // kSeqScatter, optional (slab_flags[0] == nullptr: none): per destination slab r, a counter
  // to which every epilogue warp adds, with a system-scope release after its stores, the
  // number of rows it stored into dest[r].
  unsigned int *slab_flags[kMaxRanks];
  int B, H, S, D, P;       // H = heads held by this call (the rank's heads); S = query rows
  int S_kv;                // key/value rows (= S except for partial attention over a shard)
  int H_dest;              // heads per destination row (all heads of the layer)
  int head_offset;         // global index of this call's first head
  int S_local;             // S / P
  int n_kv;                // ceil(S_kv / 128), >= 1
  int n_pairs;             // ceil(S / 256): work items per (b, h)
  int n_items;             // B * H * n_pairs
  float scale_log2;        // softmax scale * log2(e)
  int *status;
  long long wait_limit_ns;
  // Self-test only (-1 otherwise): the TMA producer of every CTA stops before its fill number
  // stall_fill (Q and K/V tile fills counted together), as if a copy never arrived, and the
  // other roles' bounded waits then run out.
  int stall_fill;
};

// Host launchers (attn.cu).
cudaError_t launch_attention(const AttnParams &p, int epilogue, cudaStream_t stream);
size_t attention_smem_bytes(int dch);

// ---------------------------------------------------------------- exchange / probe
struct RelayoutParams {
  const void *src;
  void *dest[kMaxRanks];
  int B, H, S, D, P, S_local;
};
cudaError_t launch_relayout(const RelayoutParams &p, cudaStream_t stream);

struct PreRelayoutParams {
  const void *src[kMaxRanks];  // P sequence-shard slabs [B, S/P, H_total, D]
  void *dst;                   // head-major [B, H_local, S, D]
  int B, H_total, H_local, head_offset, S, D, P, S_local;
};
cudaError_t launch_pre_relayout(const PreRelayoutParams &p, cudaStream_t stream);

struct BurstParams {
  uint4 *scratch;
  long long scratch_chunks;  // 16-byte chunks in scratch
  long long share_chunks;    // chunks per producer per burst
  int producers;
  int n_bursts;
  long long gap_iters;       // dependent FMAs per thread after each burst
  unsigned long long *stamps;
};
cudaError_t launch_burst_probe(const BurstParams &p, int threads, cudaStream_t stream);

// Allocation-free probe: device address of the fixed scratch array in the current context
// (looked up on every call), and its size.
constexpr long long kStaticProbeScratchBytes = 32LL << 20;
cudaError_t static_probe_scratch(uint4 **out);

cudaError_t launch_wait_selftest(int *status, long long limit_ns, cudaStream_t stream);

// Consumer side of the per-slab arrival counters: one thread polls *flag (acquire, system
// scope) until it has reached target (wrap-around safe), or writes XS_ERR_TIMEOUT to *status
// after limit_ns.
cudaError_t launch_slab_wait(const unsigned int *flag, unsigned int target, long long limit_ns,
                             int *status, cudaStream_t stream);

// ---------------------------------------------------------------- log-sum-exp merge
constexpr int kMaxParts = 16;
struct MergeParams {
  const float *o[kMaxParts];    // n partial outputs [rows, D] fp32
  const float *lse[kMaxParts];  // n log-sum-exps [rows] fp32 (-inf = empty part)
  int n;
  void *out;                    // [rows, D] bf16
  float *lse_out;               // [rows] fp32, nullable
  long long rows;
  int D;
};
cudaError_t launch_lse_merge(const MergeParams &p, cudaStream_t stream);
// Result of partial attention over zero keys: o = 0, lse = -inf for `rows` rows of D.
cudaError_t launch_partial_empty(float *o, float *lse, long long rows, int D, cudaStream_t stream);

int device_sm_count();

// The detail string xs_last_error_detail() returns on this thread: record_error sets it
// (printf-style) and returns `code`; clear_error empties it.
int record_error(int code, const char *fmt, ...);
void clear_error();

}  // namespace xs
