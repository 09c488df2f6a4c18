// api.cu -- the C ABI of libxs.so (declared in include/xs.h): argument checks, TMA tensor
// maps and kernel launches.  No device memory is allocated, freed or kept here, and nothing
// synchronises: every call only enqueues work on the caller's stream.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "xs.h"
#include "xs_internal.cuh"

namespace xs {
thread_local char g_detail[512] = "";

int record_error(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return code;
}

void clear_error() { g_detail[0] = '\0'; }
}  // namespace xs

namespace {

template <typename... A>
xs_status fail(xs_status code, const char *fmt, A... args) {
  return static_cast<xs_status>(xs::record_error(code, fmt, args...));
}

xs_status ok() {
  xs::clear_error();
  return XS_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

// ------------------------------------------------------------------ driver entry point
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// 3-D view {D, S, B*H} of a [B, H, S, D] bf16 tensor; box {64, 128, 1}; 128-byte swizzle;
// out-of-range elements (D padding, rows past S) read as zero.
// `rows` is the S extent of the view (the key count for k and v of a partial attention).
bool make_qkv_map(CUtensorMap *m, const void *ptr, const xs_shape &s, int rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(s.D), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(s.B) * static_cast<cuuint64_t>(s.H)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(s.D) * 2,
                           static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(s.D) * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

xs_status check_shape(const xs_shape &s, bool need_ranks) {
  if (s.B <= 0 || s.H <= 0 || s.S <= 0 || s.D <= 0 || s.P <= 0)
    return fail(XS_ERR_INVALID_ARG, "non-positive size in shape B=%d H=%d S=%d D=%d P=%d", s.B, s.H,
                s.S, s.D, s.P);
  if (s.D % 8 != 0 || s.D > 128)
    return fail(XS_ERR_UNSUPPORTED, "head dim D=%d unsupported (need D %% 8 == 0, 8 <= D <= 128)", s.D);
  if (s.P > XS_MAX_RANKS)
    return fail(XS_ERR_UNSUPPORTED, "P=%d exceeds XS_MAX_RANKS=%d", s.P, XS_MAX_RANKS);
  if (need_ranks && (s.H % s.P != 0 || s.S % s.P != 0))
    return fail(XS_ERR_UNSUPPORTED, "Ulysses sharding needs H %% P == 0 and S %% P == 0 (H=%d S=%d P=%d)",
                s.H, s.S, s.P);
  const long long elems = static_cast<long long>(s.B) * s.H * s.S * s.D;
  if (elems <= 0 || elems > (1LL << 40))
    return fail(XS_ERR_UNSUPPORTED, "tensor of %lld elements out of range", elems);
  if (static_cast<long long>(s.B) * s.H * ((s.S + 255) / 256) > 0x7fffffffLL)
    return fail(XS_ERR_UNSUPPORTED, "too many work items");
  return XS_OK;
}

xs_status check_inputs(const void *q, const void *k, const void *v, const xs_shape &s) {
  if (!q || !k || !v) return fail(XS_ERR_INVALID_ARG, "q, k and v must be non-null device pointers");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v))
    return fail(XS_ERR_INVALID_ARG, "q, k and v must be 16-byte aligned");
  (void)s;
  return XS_OK;
}

xs_status check_dest(void *const *dest, const xs_shape &s, const void *const *inputs, int n_inputs,
                     int heads_total = -1) {
  if (!dest) return fail(XS_ERR_INVALID_ARG, "dest must be a host array of P device pointers");
  const int hd = heads_total > 0 ? heads_total : s.H;
  const uintptr_t slab = static_cast<uintptr_t>(s.B) * (s.S / s.P) * hd * s.D * 2;
  const uintptr_t full = static_cast<uintptr_t>(s.B) * s.H * s.S * s.D * 2;
  for (int r = 0; r < s.P; ++r) {
    if (!dest[r]) return fail(XS_ERR_INVALID_ARG, "dest[%d] is null", r);
    if (!aligned16(dest[r])) return fail(XS_ERR_INVALID_ARG, "dest[%d] is not 16-byte aligned", r);
    const Range a{reinterpret_cast<uintptr_t>(dest[r]), reinterpret_cast<uintptr_t>(dest[r]) + slab};
    for (int o = 0; o < r; ++o) {
      const Range b{reinterpret_cast<uintptr_t>(dest[o]), reinterpret_cast<uintptr_t>(dest[o]) + slab};
      if (overlap(a, b)) return fail(XS_ERR_INVALID_ARG, "dest[%d] overlaps dest[%d]", r, o);
    }
    for (int i = 0; i < n_inputs; ++i) {
      const Range b{reinterpret_cast<uintptr_t>(inputs[i]), reinterpret_cast<uintptr_t>(inputs[i]) + full};
      if (overlap(a, b)) return fail(XS_ERR_INVALID_ARG, "dest[%d] overlaps an input tensor", r);
    }
  }
  return XS_OK;
}

// s_kv: key/value rows (-1: the same as the query rows s.S).
xs_status fill_attention(xs::AttnParams &p, const void *q, const void *k, const void *v,
                         const xs_shape &s, float scale, int *dev_status, int s_kv = -1) {
  std::memset(&p, 0, sizeof(p));
  if (s_kv < 0) s_kv = s.S;
  if (!make_qkv_map(&p.tm_q, q, s, s.S) || !make_qkv_map(&p.tm_k, k, s, s_kv) ||
      !make_qkv_map(&p.tm_v, v, s, s_kv))
    return fail(XS_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point %s)",
                encode_fn() ? "found" : "missing");
  p.B = s.B;
  p.H = s.H;
  p.S = s.S;
  p.D = s.D;
  p.P = s.P;
  p.H_dest = s.H;
  p.head_offset = 0;
  p.S_kv = s_kv;
  p.S_local = s.S / s.P;
  p.n_kv = (s_kv + 127) / 128;
  p.n_pairs = (s.S + 255) / 256;
  p.n_items = s.B * s.H * p.n_pairs;
  const double sc = scale > 0.f ? static_cast<double>(scale) : 1.0 / std::sqrt(static_cast<double>(s.D));
  p.scale_log2 = static_cast<float>(sc * 1.4426950408889634);  // scale * log2(e)
  p.status = dev_status;
  p.wait_limit_ns = xs::kWaitLimitNs;
  p.stall_fill = -1;  // never (the self-test entry point alone sets it)
  return XS_OK;
}

xs_status launched(cudaError_t e, const char *what) {
  if (e != cudaSuccess) return fail(XS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return ok();
}

}  // namespace

namespace xs {
int device_sm_count() {
  // Per-device cache; threads that race on a first call both store the same count.
  static std::atomic<int> cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}
}  // namespace xs

extern "C" {

xs_status xs_attn_a2a_fused(const void *q, const void *k, const void *v, void *const *dest,
                            xs_shape shape, float scale, xs_stream_t stream, int *dev_status) {
  xs_status st = check_shape(shape, true);
  if (st != XS_OK) return st;
  if ((st = check_inputs(q, k, v, shape)) != XS_OK) return st;
  const void *ins[3] = {q, k, v};
  if ((st = check_dest(dest, shape, ins, 3)) != XS_OK) return st;
  xs::AttnParams p;
  if ((st = fill_attention(p, q, k, v, shape, scale, dev_status)) != XS_OK) return st;
  for (int r = 0; r < shape.P; ++r) p.dest[r] = dest[r];
  return launched(xs::launch_attention(p, xs::kSeqScatter, reinterpret_cast<cudaStream_t>(stream)),
                  "attention launch");
}

xs_status xs_attn_a2a_fused_spans(const void *q, const void *k, const void *v, void *const *dest,
                                  xs_shape shape, float scale, unsigned long long *spans,
                                  long long spans_len, xs_stream_t stream, int *dev_status) {
  xs_status st = check_shape(shape, true);
  if (st != XS_OK) return st;
  if ((st = check_inputs(q, k, v, shape)) != XS_OK) return st;
  const void *ins[3] = {q, k, v};
  if ((st = check_dest(dest, shape, ins, 3)) != XS_OK) return st;
  xs::AttnParams p;
  if ((st = fill_attention(p, q, k, v, shape, scale, dev_status)) != XS_OK) return st;
  const long long need = static_cast<long long>(p.n_items) * 2 * 4 * 3;
  if (!spans || (reinterpret_cast<uintptr_t>(spans) & 7u))
    return fail(XS_ERR_INVALID_ARG, "spans must be an 8-byte aligned device pointer");
  if (spans_len < need)
    return fail(XS_ERR_INVALID_ARG, "spans holds %lld words, the call needs %lld (work items x 2 x 4 x 3)",
                spans_len, need);
  {
    const Range rs{reinterpret_cast<uintptr_t>(spans), reinterpret_cast<uintptr_t>(spans) + need * 8};
    const uintptr_t full = static_cast<uintptr_t>(shape.B) * shape.H * shape.S * shape.D * 2;
    const uintptr_t slab = full / shape.P;
    for (const void *in : {q, k, v}) {
      const Range r{reinterpret_cast<uintptr_t>(in), reinterpret_cast<uintptr_t>(in) + full};
      if (overlap(rs, r)) return fail(XS_ERR_INVALID_ARG, "spans overlaps an input tensor");
    }
    for (int r = 0; r < shape.P; ++r) {
      const Range d{reinterpret_cast<uintptr_t>(dest[r]), reinterpret_cast<uintptr_t>(dest[r]) + slab};
      if (overlap(rs, d)) return fail(XS_ERR_INVALID_ARG, "spans overlaps dest[%d]", r);
    }
  }
  for (int r = 0; r < shape.P; ++r) p.dest[r] = dest[r];
  p.spans = spans;
  return launched(xs::launch_attention(p, xs::kSeqScatterSpans, reinterpret_cast<cudaStream_t>(stream)),
                  "attention launch");
}

xs_status xs_attn_a2a_fused_rank(const void *q, const void *k, const void *v, void *const *dest,
                                 xs_shape shape, int heads_total, int head_offset, float scale,
                                 xs_stream_t stream, int *dev_status) {
  // Per-rank form: shape.H heads of this rank; H % P is not required here (the layer's
  // heads_total is), the destination rows hold heads_total heads.
  xs_shape layer = shape;
  layer.H = heads_total;
  xs_status st = check_shape(layer, true);
  if (st != XS_OK) return st;
  if ((st = check_shape(shape, false)) != XS_OK) return st;
  if (shape.S % shape.P != 0)
    return fail(XS_ERR_UNSUPPORTED, "S %% P != 0 (S=%d P=%d)", shape.S, shape.P);
  if (head_offset < 0 || shape.H > heads_total || head_offset > heads_total - shape.H)
    return fail(XS_ERR_INVALID_ARG, "heads [%d, %d) are not inside the layer's %d heads", head_offset,
                head_offset + shape.H, heads_total);
  if ((st = check_inputs(q, k, v, shape)) != XS_OK) return st;
  const void *ins[3] = {q, k, v};
  if ((st = check_dest(dest, shape, ins, 3, heads_total)) != XS_OK) return st;
  xs::AttnParams p;
  if ((st = fill_attention(p, q, k, v, shape, scale, dev_status)) != XS_OK) return st;
  p.H_dest = heads_total;
  p.head_offset = head_offset;
  for (int r = 0; r < shape.P; ++r) p.dest[r] = dest[r];
  return launched(xs::launch_attention(p, xs::kSeqScatter, reinterpret_cast<cudaStream_t>(stream)),
                  "attention launch");
}

xs_status xs_attn_a2a_fused_flags(const void *q, const void *k, const void *v, void *const *dest,
                                  unsigned int *const *slab_flags, xs_shape shape, int heads_total,
                                  int head_offset, float scale, xs_stream_t stream,
                                  int *dev_status) {
  if (!slab_flags) return fail(XS_ERR_INVALID_ARG, "slab_flags must be a host array of P device pointers");
  for (int r = 0; r < shape.P && r < XS_MAX_RANKS; ++r) {
    if (!slab_flags[r] || (reinterpret_cast<uintptr_t>(slab_flags[r]) & 3u))
      return fail(XS_ERR_INVALID_ARG, "slab_flags[%d] must be a 4-byte aligned device pointer", r);
    for (int o = 0; o < r; ++o)
      if (slab_flags[o] == slab_flags[r])
        return fail(XS_ERR_INVALID_ARG, "slab_flags[%d] and slab_flags[%d] are the same counter", o, r);
  }
  xs_shape layer = shape;
  layer.H = heads_total;
  xs_status st = check_shape(layer, true);
  if (st != XS_OK) return st;
  if ((st = check_shape(shape, false)) != XS_OK) return st;
  if (head_offset < 0 || shape.H > heads_total || head_offset > heads_total - shape.H)
    return fail(XS_ERR_INVALID_ARG, "heads [%d, %d) are not inside the layer's %d heads", head_offset,
                head_offset + shape.H, heads_total);
  if ((st = check_inputs(q, k, v, shape)) != XS_OK) return st;
  const void *ins[3] = {q, k, v};
  if ((st = check_dest(dest, shape, ins, 3, heads_total)) != XS_OK) return st;
  {
    // a counter inside a slab or an input would be overwritten by the data it counts
    const uintptr_t slab = static_cast<uintptr_t>(shape.B) * (shape.S / shape.P) * heads_total * shape.D * 2;
    const uintptr_t full = static_cast<uintptr_t>(shape.B) * shape.H * shape.S * shape.D * 2;
    for (int r = 0; r < shape.P; ++r) {
      const Range f{reinterpret_cast<uintptr_t>(slab_flags[r]), reinterpret_cast<uintptr_t>(slab_flags[r]) + 4};
      for (int o = 0; o < shape.P; ++o) {
        const Range d{reinterpret_cast<uintptr_t>(dest[o]), reinterpret_cast<uintptr_t>(dest[o]) + slab};
        if (overlap(f, d)) return fail(XS_ERR_INVALID_ARG, "slab_flags[%d] lies inside dest[%d]", r, o);
      }
      for (const void *in : {q, k, v}) {
        const Range i{reinterpret_cast<uintptr_t>(in), reinterpret_cast<uintptr_t>(in) + full};
        if (overlap(f, i)) return fail(XS_ERR_INVALID_ARG, "slab_flags[%d] lies inside an input", r);
      }
    }
  }
  xs::AttnParams p;
  if ((st = fill_attention(p, q, k, v, shape, scale, dev_status)) != XS_OK) return st;
  p.H_dest = heads_total;
  p.head_offset = head_offset;
  for (int r = 0; r < shape.P; ++r) {
    p.dest[r] = dest[r];
    p.slab_flags[r] = slab_flags[r];
  }
  return launched(xs::launch_attention(p, xs::kSeqScatter, reinterpret_cast<cudaStream_t>(stream)),
                  "attention launch");
}

xs_status xs_slab_wait(const unsigned int *flag, unsigned int target, long long limit_ns,
                       xs_stream_t stream, int *dev_status) {
  if (!flag || (reinterpret_cast<uintptr_t>(flag) & 3u))
    return fail(XS_ERR_INVALID_ARG, "flag must be a 4-byte aligned device pointer");
  if (!dev_status) return fail(XS_ERR_INVALID_ARG, "dev_status is required");
  if (limit_ns < 1000 || limit_ns > 100000000000LL)
    return fail(XS_ERR_INVALID_ARG, "limit_ns out of range [1e3, 1e11]");
  return launched(xs::launch_slab_wait(flag, target, limit_ns, dev_status, reinterpret_cast<cudaStream_t>(stream)),
                  "slab wait launch");
}

xs_status xs_attn(const void *q, const void *k, const void *v, void *out, xs_shape shape,
                  float scale, xs_stream_t stream, int *dev_status) {
  xs_status st = check_shape(shape, false);
  if (st != XS_OK) return st;
  if ((st = check_inputs(q, k, v, shape)) != XS_OK) return st;
  if (!out || !aligned16(out)) return fail(XS_ERR_INVALID_ARG, "out must be a 16-byte aligned device pointer");
  {
    const uintptr_t full = static_cast<uintptr_t>(shape.B) * shape.H * shape.S * shape.D * 2;
    const Range o{reinterpret_cast<uintptr_t>(out), reinterpret_cast<uintptr_t>(out) + full};
    for (const void *in : {q, k, v}) {
      const Range r{reinterpret_cast<uintptr_t>(in), reinterpret_cast<uintptr_t>(in) + full};
      if (overlap(o, r)) return fail(XS_ERR_INVALID_ARG, "out overlaps an input tensor");
    }
  }
  xs::AttnParams p;
  if ((st = fill_attention(p, q, k, v, shape, scale, dev_status)) != XS_OK) return st;
  p.out = out;
  return launched(xs::launch_attention(p, xs::kHeadMajor, reinterpret_cast<cudaStream_t>(stream)),
                  "attention launch");
}

xs_status xs_attn_partial(const void *q, const void *k, const void *v, float *o_part, float *lse,
                          xs_shape shape, int s_kv, float scale, xs_stream_t stream, int *dev_status) {
  if (shape.P != 1) return fail(XS_ERR_INVALID_ARG, "partial attention takes shape.P == 1 (got %d)", shape.P);
  xs_status st = check_shape(shape, false);
  if (st != XS_OK) return st;
  if (s_kv < 0) return fail(XS_ERR_INVALID_ARG, "negative key count s_kv=%d", s_kv);
  if (static_cast<long long>(shape.B) * shape.H * s_kv * shape.D > (1LL << 40))
    return fail(XS_ERR_UNSUPPORTED, "key/value shard of %d rows out of range", s_kv);
  if (!q || !aligned16(q)) return fail(XS_ERR_INVALID_ARG, "q must be a 16-byte aligned device pointer");
  if (s_kv > 0 && (!k || !v || !aligned16(k) || !aligned16(v)))
    return fail(XS_ERR_INVALID_ARG, "k and v must be 16-byte aligned device pointers");
  if (!o_part || !aligned16(o_part)) return fail(XS_ERR_INVALID_ARG, "o_part must be a 16-byte aligned device pointer");
  if (!lse || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(XS_ERR_INVALID_ARG, "lse must be a 4-byte aligned device pointer");
  const uintptr_t rows = static_cast<uintptr_t>(shape.B) * shape.H * shape.S;
  const Range ro{reinterpret_cast<uintptr_t>(o_part), reinterpret_cast<uintptr_t>(o_part) + rows * shape.D * 4};
  const Range rl{reinterpret_cast<uintptr_t>(lse), reinterpret_cast<uintptr_t>(lse) + rows * 4};
  if (overlap(ro, rl)) return fail(XS_ERR_INVALID_ARG, "o_part overlaps lse");
  {
    const Range rq{reinterpret_cast<uintptr_t>(q), reinterpret_cast<uintptr_t>(q) + rows * shape.D * 2};
    const uintptr_t kv_bytes = static_cast<uintptr_t>(shape.B) * shape.H * s_kv * shape.D * 2;
    for (const Range &o : {ro, rl}) {
      if (overlap(o, rq)) return fail(XS_ERR_INVALID_ARG, "an output overlaps q");
      for (const void *in : {k, v}) {
        if (s_kv == 0) break;
        const Range r{reinterpret_cast<uintptr_t>(in), reinterpret_cast<uintptr_t>(in) + kv_bytes};
        if (overlap(o, r)) return fail(XS_ERR_INVALID_ARG, "an output overlaps k or v");
      }
    }
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (s_kv == 0)
    return launched(xs::launch_partial_empty(o_part, lse, static_cast<long long>(rows), shape.D, s),
                    "empty-shard fill launch");
  xs::AttnParams p;
  if ((st = fill_attention(p, q, k, v, shape, scale, dev_status, s_kv)) != XS_OK) return st;
  p.out = o_part;
  p.lse = lse;
  return launched(xs::launch_attention(p, xs::kPartial, s), "partial attention launch");
}

xs_status xs_lse_merge(const float *const *o_parts, const float *const *lse_parts, int n_parts,
                       void *out, float *lse_out, long long rows, int D, xs_stream_t stream) {
  if (n_parts < 1 || n_parts > XS_MAX_PARTS)
    return fail(XS_ERR_UNSUPPORTED, "n_parts=%d outside [1, %d]", n_parts, XS_MAX_PARTS);
  if (rows < 1 || rows > (1LL << 36)) return fail(XS_ERR_INVALID_ARG, "rows=%lld out of range", rows);
  if (D < 8 || D % 8 != 0 || D > 4096)
    return fail(XS_ERR_UNSUPPORTED, "D=%d unsupported (need D %% 8 == 0, 8 <= D <= 4096)", D);
  if (!o_parts || !lse_parts) return fail(XS_ERR_INVALID_ARG, "o_parts and lse_parts must be host arrays");
  if (!out || !aligned16(out)) return fail(XS_ERR_INVALID_ARG, "out must be a 16-byte aligned device pointer");
  if (lse_out && (reinterpret_cast<uintptr_t>(lse_out) & 3u))
    return fail(XS_ERR_INVALID_ARG, "lse_out must be 4-byte aligned");
  const Range ro{reinterpret_cast<uintptr_t>(out), reinterpret_cast<uintptr_t>(out) + rows * D * 2};
  const Range rlo{reinterpret_cast<uintptr_t>(lse_out),
                  reinterpret_cast<uintptr_t>(lse_out) + (lse_out ? rows * 4 : 0)};
  if (lse_out && overlap(ro, rlo)) return fail(XS_ERR_INVALID_ARG, "out overlaps lse_out");
  xs::MergeParams p;
  std::memset(&p, 0, sizeof(p));
  for (int t = 0; t < n_parts; ++t) {
    if (!o_parts[t] || !aligned16(o_parts[t]))
      return fail(XS_ERR_INVALID_ARG, "o_parts[%d] must be a 16-byte aligned device pointer", t);
    if (!lse_parts[t] || (reinterpret_cast<uintptr_t>(lse_parts[t]) & 3u))
      return fail(XS_ERR_INVALID_ARG, "lse_parts[%d] must be a 4-byte aligned device pointer", t);
    const Range a{reinterpret_cast<uintptr_t>(o_parts[t]), reinterpret_cast<uintptr_t>(o_parts[t]) + rows * D * 4};
    const Range b{reinterpret_cast<uintptr_t>(lse_parts[t]), reinterpret_cast<uintptr_t>(lse_parts[t]) + rows * 4};
    if (overlap(a, ro) || overlap(b, ro) || (lse_out && (overlap(a, rlo) || overlap(b, rlo))))
      return fail(XS_ERR_INVALID_ARG, "part %d overlaps an output", t);
    p.o[t] = o_parts[t];
    p.lse[t] = lse_parts[t];
  }
  p.n = n_parts;
  p.out = out;
  p.lse_out = lse_out;
  p.rows = rows;
  p.D = D;
  return launched(xs::launch_lse_merge(p, reinterpret_cast<cudaStream_t>(stream)), "merge launch");
}

xs_status xs_a2a_relayout(const void *src, void *const *dest, xs_shape shape, xs_stream_t stream) {
  // Any H: the pack step of a GPU that holds only H/N of the layer's heads uses it too.
  xs_status st = check_shape(shape, false);
  if (st != XS_OK) return st;
  if (shape.S % shape.P != 0)
    return fail(XS_ERR_UNSUPPORTED, "S %% P != 0 (S=%d P=%d)", shape.S, shape.P);
  if (!src || !aligned16(src)) return fail(XS_ERR_INVALID_ARG, "src must be a 16-byte aligned device pointer");
  const void *ins[1] = {src};
  if ((st = check_dest(dest, shape, ins, 1)) != XS_OK) return st;
  xs::RelayoutParams p;
  std::memset(&p, 0, sizeof(p));
  p.src = src;
  for (int r = 0; r < shape.P; ++r) p.dest[r] = dest[r];
  p.B = shape.B;
  p.H = shape.H;
  p.S = shape.S;
  p.D = shape.D;
  p.P = shape.P;
  p.S_local = shape.S / shape.P;
  return launched(xs::launch_relayout(p, reinterpret_cast<cudaStream_t>(stream)), "relayout launch");
}

xs_status xs_a2a_pre(void *const *src, void *dst, xs_shape shape, int heads_local, int head_offset,
                     xs_stream_t stream) {
  xs_status st = check_shape(shape, true);
  if (st != XS_OK) return st;
  if (heads_local <= 0 || head_offset < 0 || head_offset > shape.H - heads_local)
    return fail(XS_ERR_INVALID_ARG, "heads [%d, %d) are not inside the layer's %d heads", head_offset,
                head_offset + heads_local, shape.H);
  if (!dst || !aligned16(dst)) return fail(XS_ERR_INVALID_ARG, "dst must be a 16-byte aligned device pointer");
  if (!src) return fail(XS_ERR_INVALID_ARG, "src must be a host array of P device pointers");
  const uintptr_t slab = static_cast<uintptr_t>(shape.B) * (shape.S / shape.P) * shape.H * shape.D * 2;
  const uintptr_t out_bytes = static_cast<uintptr_t>(shape.B) * heads_local * shape.S * shape.D * 2;
  const Range o{reinterpret_cast<uintptr_t>(dst), reinterpret_cast<uintptr_t>(dst) + out_bytes};
  xs::PreRelayoutParams p;
  std::memset(&p, 0, sizeof(p));
  for (int r = 0; r < shape.P; ++r) {
    if (!src[r] || !aligned16(src[r])) return fail(XS_ERR_INVALID_ARG, "src[%d] is null or not 16-byte aligned", r);
    const Range a{reinterpret_cast<uintptr_t>(src[r]), reinterpret_cast<uintptr_t>(src[r]) + slab};
    if (overlap(a, o)) return fail(XS_ERR_INVALID_ARG, "src[%d] overlaps dst", r);
    p.src[r] = src[r];
  }
  p.dst = dst;
  p.B = shape.B;
  p.H_total = shape.H;
  p.H_local = heads_local;
  p.head_offset = head_offset;
  p.S = shape.S;
  p.D = shape.D;
  p.P = shape.P;
  p.S_local = shape.S / shape.P;
  return launched(xs::launch_pre_relayout(p, reinterpret_cast<cudaStream_t>(stream)), "pre-exchange launch");
}

xs_status xs_burst_probe(void *scratch, long long scratch_bytes, xs_burst_cfg cfg,
                         unsigned long long *stamps, xs_stream_t stream) {
  if (!scratch || !stamps || !aligned16(scratch) || (reinterpret_cast<uintptr_t>(stamps) & 7u))
    return fail(XS_ERR_INVALID_ARG, "scratch (16-byte aligned) and stamps (8-byte aligned) are required");
  if (cfg.producers < 1 || cfg.producers > 4096 || cfg.n_bursts < 1 || cfg.n_bursts > (1 << 20) ||
      cfg.gap_cycles < 0 || cfg.gap_cycles > (1LL << 30) || cfg.burst_bytes <= 0 || scratch_bytes < 16 ||
      cfg.threads_per_producer < 32 || cfg.threads_per_producer > 1024 || cfg.threads_per_producer % 32)
    return fail(XS_ERR_INVALID_ARG, "burst probe configuration out of range");
  if (cfg.burst_bytes % (16LL * cfg.producers) != 0)
    return fail(XS_ERR_INVALID_ARG, "burst_bytes must be a multiple of 16 * producers");
  const long long share = cfg.burst_bytes / 16 / cfg.producers;
  if (share * cfg.producers > scratch_bytes / 16)
    return fail(XS_ERR_INVALID_ARG, "one burst (%lld bytes) exceeds the scratch buffer", cfg.burst_bytes);
  const Range a{reinterpret_cast<uintptr_t>(scratch), reinterpret_cast<uintptr_t>(scratch) + scratch_bytes};
  const Range b{reinterpret_cast<uintptr_t>(stamps),
                reinterpret_cast<uintptr_t>(stamps) + 32ull * cfg.producers * cfg.n_bursts};
  if (overlap(a, b)) return fail(XS_ERR_INVALID_ARG, "stamps overlaps scratch");
  xs::BurstParams p;
  p.scratch = static_cast<uint4 *>(scratch);
  p.scratch_chunks = scratch_bytes / 16;
  p.share_chunks = share;
  p.producers = cfg.producers;
  p.n_bursts = cfg.n_bursts;
  p.gap_iters = cfg.gap_cycles / 4;  // one dependent FMA is about 4 cycles
  p.stamps = stamps;
  return launched(xs::launch_burst_probe(p, cfg.threads_per_producer, reinterpret_cast<cudaStream_t>(stream)),
                  "burst probe launch");
}

xs_status xs_burst_probe_static(xs_burst_cfg cfg, unsigned long long *stamps, xs_stream_t stream) {
  if (!stamps || (reinterpret_cast<uintptr_t>(stamps) & 7u))
    return fail(XS_ERR_INVALID_ARG, "stamps (8-byte aligned device pointer) is required");
  if (cfg.producers < 1 || cfg.producers > 4096 || cfg.n_bursts < 1 || cfg.n_bursts > (1 << 20) ||
      cfg.gap_cycles < 0 || cfg.gap_cycles > (1LL << 30) || cfg.burst_bytes <= 0 ||
      cfg.threads_per_producer < 32 || cfg.threads_per_producer > 1024 || cfg.threads_per_producer % 32)
    return fail(XS_ERR_INVALID_ARG, "burst probe configuration out of range");
  if (cfg.burst_bytes % (16LL * cfg.producers) != 0)
    return fail(XS_ERR_INVALID_ARG, "burst_bytes must be a multiple of 16 * producers");
  if (cfg.burst_bytes > XS_BURST_STATIC_SCRATCH_BYTES)
    return fail(XS_ERR_UNSUPPORTED,
                "burst of %lld bytes exceeds the fixed %lld-byte scratch of xs_burst_probe_static; "
                "use xs_burst_probe with a caller-allocated buffer",
                cfg.burst_bytes, static_cast<long long>(XS_BURST_STATIC_SCRATCH_BYTES));
  static_assert(XS_BURST_STATIC_SCRATCH_BYTES == xs::kStaticProbeScratchBytes, "scratch size mismatch");
  static_assert(XS_MAX_PARTS == xs::kMaxParts, "part count mismatch");
  uint4 *scratch = nullptr;
  cudaError_t e = xs::static_probe_scratch(&scratch);
  if (e != cudaSuccess) return fail(XS_ERR_CUDA, "scratch address lookup: %s", cudaGetErrorString(e));
  xs::BurstParams p;
  p.scratch = scratch;
  p.scratch_chunks = XS_BURST_STATIC_SCRATCH_BYTES / 16;
  p.share_chunks = cfg.burst_bytes / 16 / cfg.producers;
  p.producers = cfg.producers;
  p.n_bursts = cfg.n_bursts;
  p.gap_iters = cfg.gap_cycles / 4;
  p.stamps = stamps;
  return launched(xs::launch_burst_probe(p, cfg.threads_per_producer, reinterpret_cast<cudaStream_t>(stream)),
                  "burst probe launch");
}

xs_status xs_selftest_bounded_wait(int *dev_status, long long limit_ns, xs_stream_t stream) {
  if (!dev_status) return fail(XS_ERR_INVALID_ARG, "dev_status is required");
  if (limit_ns < 1000 || limit_ns > 10000000000LL)
    return fail(XS_ERR_INVALID_ARG, "limit_ns out of range [1e3, 1e10]");
  return launched(xs::launch_wait_selftest(dev_status, limit_ns, reinterpret_cast<cudaStream_t>(stream)),
                  "self-test launch");
}

xs_status xs_selftest_attn_abort(const void *q, const void *k, const void *v, void *out,
                                 xs_shape shape, int stall_fill, long long limit_ns,
                                 xs_stream_t stream, int *dev_status) {
  if (!dev_status) return fail(XS_ERR_INVALID_ARG, "dev_status is required");
  if (stall_fill < 0) return fail(XS_ERR_INVALID_ARG, "stall_fill must be >= 0 (got %d)", stall_fill);
  if (limit_ns < 1000 || limit_ns > 10000000000LL)
    return fail(XS_ERR_INVALID_ARG, "limit_ns out of range [1e3, 1e10]");
  xs_status st = check_shape(shape, false);
  if (st != XS_OK) return st;
  if ((st = check_inputs(q, k, v, shape)) != XS_OK) return st;
  if (!out || !aligned16(out)) return fail(XS_ERR_INVALID_ARG, "out must be a 16-byte aligned device pointer");
  {
    const uintptr_t full = static_cast<uintptr_t>(shape.B) * shape.H * shape.S * shape.D * 2;
    const Range o{reinterpret_cast<uintptr_t>(out), reinterpret_cast<uintptr_t>(out) + full};
    for (const void *in : {q, k, v}) {
      const Range r{reinterpret_cast<uintptr_t>(in), reinterpret_cast<uintptr_t>(in) + full};
      if (overlap(o, r)) return fail(XS_ERR_INVALID_ARG, "out overlaps an input tensor");
    }
  }
  xs::AttnParams p;
  if ((st = fill_attention(p, q, k, v, shape, 0.f, dev_status)) != XS_OK) return st;
  p.out = out;
  p.wait_limit_ns = limit_ns;
  p.stall_fill = stall_fill;
  return launched(xs::launch_attention(p, xs::kHeadMajor, reinterpret_cast<cudaStream_t>(stream)),
                  "attention self-test launch");
}

const char *xs_get_error_string(xs_status status) {
  switch (status) {
    case XS_OK: return "XS_OK";
    case XS_ERR_INVALID_ARG: return "XS_ERR_INVALID_ARG";
    case XS_ERR_UNSUPPORTED: return "XS_ERR_UNSUPPORTED";
    case XS_ERR_CUDA: return "XS_ERR_CUDA";
    case XS_ERR_TIMEOUT: return "XS_ERR_TIMEOUT";
  }
  return "XS_ERR_UNKNOWN";
}

int xs_version(void) { return XS_VERSION; }

const char *xs_last_error_detail(void) { return xs::g_detail; }

}  // extern "C"
