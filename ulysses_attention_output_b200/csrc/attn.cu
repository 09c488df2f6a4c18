// attn.cu -- non-causal softmax attention on sm_100a with an epilogue that either writes the
// head-major output or scatters each finished tile into the Ulysses sequence-shard slabs
// (the post-attention All-to-All fused at tile granularity).
//
// Operation: O = softmax(Q K^T * scale) V per (b, h) -- page "X-Stage: An Overlooked
// Pipeline Stage for Communication-Computation Overlap in DiT Inference", abstract and the
// explainer's "Technisches Resuemee" -> "Zentrale Beitraege" -> "FlashAttention-A2A
// (Piggybacking)": the owner of an output tile issues the stores of that tile into the
// destination rank's sequence shard and immediately resumes the next tile's loop over keys,
// which is the gap in which the issued stores drain.  No warp or SM is dedicated to the
// exchange: the same warps that ran the softmax write the tile and go on.
//
// A third epilogue writes the partial attention of the query rows over one key/value shard
// (S_kv keys) in fp32 together with each row's log-sum-exp, for the Route primitive of the
// page "Move the Query, Not the Cache: Characterizing Cross-Instance Latent Attention
// Redistribution Across GPU Fabrics" ("Methodik" -> "Primitiv-Vergleich"): the owner of a
// KV shard attends the routed queries over its keys and the requester merges the results.
//
// Structure of one persistent CTA (320 threads, one CTA per SM):
//   warps 0-3  softmax for Q tile 0 (one thread per query row = one TMEM lane)
//   warps 4-7  softmax for Q tile 1
//   warp  8    TMA producer: Q tiles once per work item, then K_j, V_j through a 3-slot ring
//   warp  9    TMEM allocator and tcgen05.mma issuer (the warp runs the loop, one elected
//              lane issues)
// A work item is 256 query rows (two 128-row tiles) of one (b, h).  Tensor memory holds
//   cols [0,128)   S0 = Q0 K^T (fp32), overwritten in place by P0 (bf16 pairs, 64 cols)
//   cols [128,256) S1 / P1
//   cols [256,384) O0 (fp32, D padded to a multiple of 16)
//   cols [384,512) O1
// The MMA issue order per key tile j is QK0(j+1), PV1(j), QK1(j+1), PV0(j+1), so each tile's
// softmax overlaps the other tile's two MMAs.  The running maximum is only moved when a new
// row maximum exceeds it by more than 32 (in the exp2 domain); P then stays below 2^32, so O
// and l stay below 2^32 * S * max|v| and 2^32 * S, far inside the fp32 range, and the rescale
// of O (done by the softmax thread itself, after the previous P V completed) is
// rare (the previous P V is complete by then: it precedes the Q K^T whose result the
// softmax has just read).  P V consumes the probabilities rounded to bf16, and l sums those same rounded values
// in fp32, so the normalised weights of every row add up to one.  The softmax works on column
// pairs in packed fp32 (f32x2) and computes 4 of every 16 pairs of exponentials with an FMA-pipe
// polynomial instead of MUFU ex2, because at one exponential per 4*D FLOPs MUFU alone would
// take as long as the tensor core.
#include <mutex>

#include "xs_internal.cuh"

namespace xs {
namespace {

constexpr int kThreads = 320;
constexpr int kStages = 3;           // K/V ring slots
constexpr int kStageRows = 16;       // rows staged per warp per epilogue round (head-major / partial)
constexpr int kChunkBytes = 16384;   // 128 rows x 128 bytes (64 bf16) per swizzle panel
// A rescale makes the whole warp reload and store O; with keys of outlying norm a threshold of
// 8 made that happen in most key tiles of some warp (4% slower on such inputs than 32).
#ifndef XS_RESCALE_LOG2
#define XS_RESCALE_LOG2 32
#endif
constexpr float kRescaleThreshold = XS_RESCALE_LOG2;  // log2 of the largest tolerated P before rescale

// TMEM column of S_t / P_t and of O_t for Q tile t.
__host__ __device__ constexpr uint32_t col_s(int t) { return 128u * static_cast<uint32_t>(t); }
__host__ __device__ constexpr uint32_t col_o(int t) { return 256u + 128u * static_cast<uint32_t>(t); }

// Shared memory layout (offsets from a 1024-byte aligned base).
template <int DCH>
struct Smem {
  static constexpr uint32_t kTile = DCH * kChunkBytes;
  static constexpr uint32_t kQ = 0;                                   // 2 tiles
  static constexpr uint32_t kKV = kQ + 2 * kTile;                     // kStages tiles
  // P_t: 128 rows x 128 keys bf16 per Q tile, two 128-byte-swizzled panels of 64 keys (the
  // A operand of P V, K-major); after a work item's last P V it holds the staging rows of the
  // head-major and partial epilogues of tile t.
  static constexpr uint32_t kP = kKV + kStages * kTile;
  static constexpr uint32_t kPTile = 2 * kChunkBytes;
  static constexpr uint32_t kStageRowBytes = DCH * 128;
  static_assert(kStageRows * kStageRowBytes <= 4096, "a warp's staging rows must fit in its 32 P rows");
  static constexpr uint32_t kRowPtr = kP + 2 * kPTile;                // 8 warps x 16 pointers
  static constexpr uint32_t kBars = kRowPtr + 8 * kStageRows * 8;
  // barriers: q_full[2] q_empty[2] kv_full[S] kv_empty[S] s_full[2] s_read[2] p_full[2]
  //           p_free[2] drain go[2][4]
  static constexpr uint32_t kNumBars = 2 + 2 + kStages + kStages + 2 + 2 + 2 + 2 + 1 + 8;
  static constexpr uint32_t kMisc = kBars + kNumBars * 8;             // tmem base, abort flag
  static constexpr uint32_t kTotal = kMisc + 16;
  static constexpr size_t kAlloc = kTotal + 1024;                     // room for alignment
};

__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }
__device__ __forceinline__ uint32_t f2u(float x) { return __float_as_uint(x); }

// Column pairs (of 64 per 128-key tile) whose exponentials run on the FMA pipe instead of
// MUFU: kEmulatedPer16 of every 16 pairs, spread evenly.
#ifndef XS_EMULATED_PER16
#define XS_EMULATED_PER16 3  // 0..8 measured with the exponential hand-over: 3 fastest (1% ahead of 4)
#endif
constexpr int kEmulatedPer16 = XS_EMULATED_PER16;
__host__ __device__ constexpr bool emulated_pair(int c) {
  return ((c * kEmulatedPer16) & 15) < kEmulatedPer16;
}

// 2^x for a pair of fp32 values on the FMA pipe (no MUFU).  Range reduction x = n + f with
// n = round-to-nearest(x) obtained by adding and subtracting 1.5 * 2^23, f in [-1/2, 1/2];
// 2^f by a degree-3 polynomial with p(0) = 1 fitted for minimax relative error (1.0e-4) by
// csrc/fit_exp2_poly.py; 2^n applied by adding n to the exponent field.  Inputs below -127
// are clamped there, which yields exactly +0; masked entries (-inf) therefore give 0.
__device__ __forceinline__ void exp2_fma_pair(uint64_t x2, float &p0, float &p1) {
  constexpr uint32_t kC1 = 0x3f317afdu, kC2 = 0x3e780627u, kC3 = 0x3d61512eu;
  float x0, x1;
  ptx::f2x_split(x2, x0, x1);
  const uint64_t x = ptx::f2x(fmaxf(x0, -127.f), fmaxf(x1, -127.f));
  const uint64_t shifter = ptx::f2x(12582912.f, 12582912.f);
  const uint64_t t = ptx::add2(x, shifter);
  const uint64_t f = ptx::sub2(x, ptx::sub2(t, shifter));
  uint64_t q = ptx::fma2(f, ptx::f2x(u2f(kC3), u2f(kC3)), ptx::f2x(u2f(kC2), u2f(kC2)));
  q = ptx::fma2(q, f, ptx::f2x(u2f(kC1), u2f(kC1)));
  q = ptx::fma2(q, f, ptx::f2x(1.f, 1.f));
  float q0, q1, t0, t1;
  ptx::f2x_split(q, q0, q1);
  ptx::f2x_split(t, t0, t1);
  // The low bits of t hold n (t = 1.5 * 2^23 + n exactly); n * 2^23 added to the bits of 2^f
  // moves its exponent by n: one integer multiply-add per element.
  p0 = u2f(ptx::mad_lo_u32(f2u(t0), 1u << 23, f2u(q0)));
  p1 = u2f(ptx::mad_lo_u32(f2u(t1), 1u << 23, f2u(q1)));
}

// acc += the two bf16 halves of pk, each converted exactly and added with one fp32 rounding
// (sm_100 mixed-precision add): two instructions per pair, no unpacking.
__device__ __forceinline__ void madd2(uint64_t &acc, uint32_t pk) {
  float a0, a1;
  ptx::f2x_split(acc, a0, a1);
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
      : "+f"(a0), "+f"(a1) : "r"(pk));
  acc = ptx::f2x(a0, a1);
}

template <int DCH, int EPI, int KSQ>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using L = Smem<DCH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t *base = smem_raw + (base_u32 - raw_u32);

  const uint32_t sQ = base_u32 + L::kQ;
  const uint32_t sKV = base_u32 + L::kKV;
  const uint32_t sP = base_u32 + L::kP;
  const uint32_t bar0 = base_u32 + L::kBars;
  // barrier addresses
  auto q_full = [&](int t) { return bar0 + 8u * (0 + t); };
  auto q_empty = [&](int t) { return bar0 + 8u * (2 + t); };
  auto kv_full = [&](uint32_t s) { return bar0 + 8u * (4 + s); };
  auto kv_empty = [&](uint32_t s) { return bar0 + 8u * (4 + kStages + s); };
  // S_t = Q_t K_j^T complete (MMA -> softmax)
  auto s_full = [&](int t) { return bar0 + 8u * (4 + 2 * kStages + t); };
  // the softmax of tile t holds S_t in registers: Q K^T of the next key tile may overwrite it
  auto s_read = [&](int t) { return bar0 + 8u * (6 + 2 * kStages + t); };
  // P_t written to shared memory (and O_t rescaled if needed): P V may run
  auto p_full = [&](int t) { return bar0 + 8u * (8 + 2 * kStages + t); };
  // P V of tile t complete: P_t may be rewritten, O_t read or rescaled (MMA -> softmax)
  auto p_free = [&](int t) { return bar0 + 8u * (10 + 2 * kStages + t); };
  const uint32_t drain_bar = bar0 + 8u * (12 + 2 * kStages);
  // go(t, q): the softmax warp of tile t and TMEM lane quadrant q may start its exponentials
  // (the other tile's warp on the same SM sub-partition has finished its own)
  auto go = [&](int t, int q) { return bar0 + 8u * (13 + 2 * kStages + 4 * t + q); };
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(base + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(base + L::kMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      ptx::mbar_init(q_full(t), 1);
      ptx::mbar_init(q_empty(t), 1);
      ptx::mbar_init(s_full(t), 1);
      ptx::mbar_init(s_read(t), 4);  // one arrival per softmax warp of the tile
      ptx::mbar_init(p_full(t), 4);
      ptx::mbar_init(p_free(t), 1);
    }
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(kv_full(s), 1);
      ptx::mbar_init(kv_empty(s), 1);
    }
    ptx::mbar_init(drain_bar, 1);
    for (int t = 0; t < 2; ++t)
      for (int q = 0; q < 4; ++q) ptx::mbar_init(go(t, q), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 9) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_holder), 512);
    ptx::tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    ptx::prefetch_tmap(&p.tm_q);
    ptx::prefetch_tmap(&p.tm_k);
    ptx::prefetch_tmap(&p.tm_v);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};
  const int n_kv = p.n_kv;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kv_it = 0, it = 0;
      int q_filled0 = -1, q_filled1 = -1;
      int fills = 0;  // Q and K/V tile fills started (self-test stall point)
      bool ok = true;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++it) {
        const int bh = item / p.n_pairs;
        const int q0 = (item - bh * p.n_pairs) * 256;
        for (int t = 0; t < 2 && ok; ++t) {
          ok = bounded_wait(q_empty(t), (it & 1u) ^ 1u, ctl) && fills++ != p.stall_fill;
          if (!ok) break;
          ptx::mbar_arrive_expect_tx(q_full(t), L::kTile);
          for (int c = 0; c < DCH; ++c)
            ptx::tma_load_3d(sQ + t * L::kTile + c * kChunkBytes, &p.tm_q, q_full(t), c * 64,
                             q0 + 128 * t, bh);
          if (t == 0) q_filled0 = static_cast<int>(it);
          else q_filled1 = static_cast<int>(it);
        }
        // K runs one key tile ahead of V: K_0, K_1, V_0, K_2, V_1, ..., K_{n-1}, V_{n-2},
        // V_{n-1} -- the order in which the MMA thread needs them (Q K_{j+1}^T before P_j V_j).
        for (int f = 0; f < 2 * n_kv && ok; ++f) {
          const bool is_k = f == 0 || (f & 1 && (f + 1) / 2 < n_kv);
          const int j = f == 0 ? 0 : is_k ? (f + 1) / 2 : (f == 2 * n_kv - 1 ? n_kv - 1 : f / 2 - 1);
          const uint32_t slot = kv_it % kStages;
          ok = bounded_wait(kv_empty(slot), ((kv_it / kStages) & 1u) ^ 1u, ctl) && fills++ != p.stall_fill;
          if (!ok) break;
          ptx::mbar_arrive_expect_tx(kv_full(slot), L::kTile);
          const CUtensorMap *tm = is_k ? &p.tm_k : &p.tm_v;
          for (int c = 0; c < DCH; ++c)
            ptx::tma_load_3d(sKV + slot * L::kTile + c * kChunkBytes, tm, kv_full(slot), c * 64,
                             j * 128, bh);
          ++kv_it;
        }
      }
      if (!ok) {
        // Abort: let every copy this thread started land before the CTA can exit.
        // The ring slots hold the last (up to) kStages fills, numbered kv_it - kStages .. kv_it - 1.
        for (uint32_t f = kv_it > kStages ? kv_it - kStages : 0; f < kv_it; ++f)
          bounded_wait_drain(kv_full(f % kStages), (f / kStages) & 1u, kDrainLimitNs);
        if (q_filled0 >= 0)
          bounded_wait_drain(q_full(0), static_cast<uint32_t>(q_filled0) & 1u, kDrainLimitNs);
        if (q_filled1 >= 0)
          bounded_wait_drain(q_full(1), static_cast<uint32_t>(q_filled1) & 1u, kDrainLimitNs);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop (waits, loop control, descriptor arithmetic, all
    // warp-uniform) and one elected lane issues each MMA and commit.  Run by lane 0 alone,
    // the same loop left the tensor core idle between MMA groups for long enough to cost
    // up to 15% in a layout with more warps per SM.
    //
    // Per key tile j the order is Q_0 K_{j+1}^T, Q_1 K_{j+1}^T (each as soon as that tile's
    // softmax has read S(j) into registers), then P_0 V_j, P_1 V_j (each as soon as that tile's
    // P(j) is in shared memory).  S of the next key tile is thus ready before the softmax of
    // the current one ends, and the softmax never waits for the tensor core's P V + Q K^T of
    // its own tile in between.
    {
      const int ks_d = (p.D + 15) >> 4;              // K steps of 16 covering the true D
      const uint32_t n_pv = static_cast<uint32_t>(ks_d * 16);   // N of P V (D padded to 16)
      const uint32_t idesc_qk = ptx::idesc_bf16_f32(128, 128, 0);
      const uint32_t idesc_pv = ptx::idesc_bf16_f32(128, n_pv, 1);
      uint32_t kv_base = 0, it = 0;
      uint32_t sr0 = 0, sr1 = 0, pc0 = 0, pc1 = 0;  // s_read / p_full phases consumed per tile
      bool ok = true;

      // Descriptors are built once; per MMA only compile-time offsets are added (a per-MMA
      // rebuild in the issue loop costs ~1.5x the MMA time of a 128x128x16 step).  Adding to
      // the start-address field never carries: shared addresses are below 2^18 bytes.
      const uint64_t dq0 = ptx::smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dk0 = ptx::smem_desc_sw128(sKV, 16, 1024);
      const uint64_t dv0 = ptx::smem_desc_sw128(sKV, kChunkBytes, 1024);
      const uint64_t dp0 = ptx::smem_desc_sw128(sP, 16, 1024);
      constexpr uint64_t kTileDesc = L::kTile >> 4;   // one Q/K/V tile, in descriptor units
      constexpr uint64_t kPDesc = L::kPTile >> 4;     // one P tile

      // KSQ K steps of 16 are issued: every K step of the padded D (DCH * 64), except in the
      // instance for D <= 80, which issues 5.  TMA fills Q and K beyond D with zeros, so the
      // steps past D add exact zeros to S.  The count is a compile-time constant; no MMA is
      // issued under a run-time condition (instances of this kernel that did so computed a
      // wrong S for D = 72 .. 112 in some builds).
      auto issue_qk = [&](int t, uint32_t slot) {
        const uint64_t a = dq0 + static_cast<uint64_t>(t) * kTileDesc;
        const uint64_t b = dk0 + static_cast<uint64_t>(slot) * kTileDesc;
        const uint32_t d = tmem + col_s(t);
#pragma unroll
        for (int ks = 0; ks < KSQ; ++ks) {
          const uint64_t off = static_cast<uint64_t>(((ks >> 2) * kChunkBytes + (ks & 3) * 32) >> 4);
          ptx::mma_ss_elect(d, a + off, b + off, idesc_qk, ks > 0 ? 1u : 0u);
        }
      };
      // O_t (+)= P_t V: A = P_t from shared memory (K-major, 128 keys in two swizzled panels),
      // B = V tile, MN-major (LBO = distance between 64-column panels, SBO = 8 key rows).
      auto issue_pv = [&](int t, uint32_t slot, bool acc) {
        const uint64_t a = dp0 + static_cast<uint64_t>(t) * kPDesc;
        const uint64_t b = dv0 + static_cast<uint64_t>(slot) * kTileDesc;
        const uint32_t d = tmem + col_o(t);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t off = static_cast<uint64_t>(((ks >> 2) * kChunkBytes + (ks & 3) * 32) >> 4);
          ptx::mma_ss_elect(d, a + off, b + static_cast<uint64_t>(ks * (2048 >> 4)), idesc_pv,
                            (acc || ks > 0) ? 1u : 0u);
        }
      };
      // Ring slot and phase parity of fill number f.  Within an item K_0 is fill 0, K_{j+1}
      // fill 2j + 1 and V_j fill 2j + 2, except V_{n-1}: fill 2n - 1 (K one key tile ahead).
      auto slot_of = [](uint32_t f) { return f % kStages; };
      auto par_of = [](uint32_t f) { return (f / kStages) & 1u; };
      // Wait (whole warp) for a barrier phase; false when the CTA aborts.
      auto wait = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, bounded_wait(bar, parity, ctl));
      };

      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++it) {
        ok = wait(q_full(0), it & 1u) && wait(q_full(1), it & 1u);
        const uint32_t fK0 = kv_base;
        ok = ok && wait(kv_full(slot_of(fK0)), par_of(fK0));
        // The previous item's last S_t must have been read before Q_t K_0^T overwrites it.
        if (ok && it > 0) ok = wait(s_read(0), sr0++ & 1u);
        if (!ok) break;
        ptx::tc_fence_after();
        issue_qk(0, slot_of(fK0));
        ptx::mma_commit_elect(s_full(0));
        if (n_kv == 1) ptx::mma_commit_elect(q_empty(0));
        if (it > 0) {
          ok = wait(s_read(1), sr1++ & 1u);
          if (!ok) break;
          ptx::tc_fence_after();
        }
        issue_qk(1, slot_of(fK0));
        ptx::mma_commit_elect(s_full(1));
        ptx::mma_commit_elect(kv_empty(slot_of(fK0)));
        if (n_kv == 1) ptx::mma_commit_elect(q_empty(1));

        for (int j = 0; j < n_kv && ok; ++j) {
          const uint32_t fV = kv_base + 2 * j + (j + 1 < n_kv ? 2 : 1);
          if (j + 1 < n_kv) {
            const uint32_t fK = kv_base + 2 * j + 1;
            ok = wait(kv_full(slot_of(fK)), par_of(fK)) && wait(s_read(0), sr0++ & 1u);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_qk(0, slot_of(fK));
            ptx::mma_commit_elect(s_full(0));
            if (j + 2 == n_kv) ptx::mma_commit_elect(q_empty(0));
            ok = wait(s_read(1), sr1++ & 1u);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_qk(1, slot_of(fK));
            ptx::mma_commit_elect(s_full(1));
            ptx::mma_commit_elect(kv_empty(slot_of(fK)));
            if (j + 2 == n_kv) ptx::mma_commit_elect(q_empty(1));
          }
          ok = wait(kv_full(slot_of(fV)), par_of(fV)) && wait(p_full(0), pc0++ & 1u);
          if (!ok) break;
          ptx::tc_fence_after();
          issue_pv(0, slot_of(fV), j > 0);
          ptx::mma_commit_elect(p_free(0));
          ok = wait(p_full(1), pc1++ & 1u);
          if (!ok) break;
          ptx::tc_fence_after();
          issue_pv(1, slot_of(fV), j > 0);
          ptx::mma_commit_elect(p_free(1));
          ptx::mma_commit_elect(kv_empty(slot_of(fV)));
        }
        kv_base += 2 * static_cast<uint32_t>(n_kv);
      }
      // Every MMA the elected lane issued must be complete before TMEM is released.
      ptx::mma_commit_elect(drain_bar);
      bounded_wait_drain(drain_bar, 0, kDrainLimitNs);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;         // Q tile of this warpgroup
    const int wq = warp & 3;         // TMEM lane quadrant
    const int row = wq * 32 + lane;  // query row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_base + col_s(t);
    const uint32_t tO = tmem + lane_base + col_o(t);
    const float sl2 = p.scale_log2;
    const int D = p.D;
    // This thread's row of P_t (two 64-key panels, 128-byte rows, 16-byte chunks XOR-swizzled
    // by row % 8, as TMA lays out a Q tile) and, after the item's last P V, the staging rows of
    // this warp: the 4 KB of panel 0 that hold the warp's own 32 P rows, so that a warp that
    // has moved on to the next item's P never writes where another still stages.
    const uint32_t sP_t = sP + static_cast<uint32_t>(t) * L::kPTile;
    const uint32_t p_row = sP_t + static_cast<uint32_t>(row) * 128u;
    const uint32_t p_sw = static_cast<uint32_t>(row & 7);
    uint8_t *stg = base + L::kP + t * L::kPTile + wq * 4096;
    uint8_t **rowptr = reinterpret_cast<uint8_t **>(base + L::kRowPtr) + warp * kStageRows;
    uint32_t sc = 0;    // s_full phases consumed
    uint32_t kx = 0;    // exponential phases of this warp so far (all items)
    uint32_t npv = 0;   // P V of this tile handed to the MMA thread (p_free completes once each)
    bool ok = true;

    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const int bh = item / p.n_pairs;
      const int q0 = (item - bh * p.n_pairs) * 256;
      float m_run = -INFINITY;  // running max in the exp2 domain (scaled)
      float l_run = 0.f;

      for (int j = 0; j < n_kv; ++j) {
        ok = bounded_wait(s_full(t), sc & 1u, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++sc;
        ptx::tc_fence_after();
        const int kv_valid = p.S_kv - j * 128;  // < 128 only on a ragged last key tile
        // Pass 1: the row's 128 scores from TMEM into registers (one round trip); S_t is then
        // free, and Q K^T of the next key tile may overwrite it while this thread computes.
        uint32_t sr[128];
#pragma unroll
        for (int q = 0; q < 4; ++q) ptx::tmem_ld32(tS + 32 * q, sr + 32 * q);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) ptx::reg_fence32(sr + 32 * q);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(s_read(t));  // one arrival per warp
        if (kv_valid < 128) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= kv_valid) sr[c] = 0xff800000u;  // -inf
        }
        float m0 = u2f(sr[0]), m1 = u2f(sr[1]), m2 = u2f(sr[2]), m3 = u2f(sr[3]);
#pragma unroll
        for (int c = 4; c < 124; c += 8) {
          m0 = ptx::max3(m0, u2f(sr[c]), u2f(sr[c + 1]));
          m1 = ptx::max3(m1, u2f(sr[c + 2]), u2f(sr[c + 3]));
          m2 = ptx::max3(m2, u2f(sr[c + 4]), u2f(sr[c + 5]));
          m3 = ptx::max3(m3, u2f(sr[c + 6]), u2f(sr[c + 7]));
        }
        m0 = ptx::max3(m0, u2f(sr[124]), u2f(sr[125]));
        m1 = ptx::max3(m1, u2f(sr[126]), u2f(sr[127]));
        const float mx = ptx::max3(m0, m1, fmaxf(m2, m3)) * sl2;
        bool rescale = false;
        float alpha = 1.f;
        if (mx > m_run + kRescaleThreshold) {
          alpha = ptx::ex2(m_run - mx);  // 0 on the first tile (m_run = -inf)
          l_run *= alpha;
          m_run = mx;
          rescale = (j > 0);
        }
        // Pass 2 from the registers of pass 1: p = 2^(s * scale * log2 e - m) in packed fp32
        // pairs, rounded to bf16 pairs (pk[i] = keys 2i, 2i + 1).  A fixed subset of the pairs
        // uses the FMA-pipe exponential instead of MUFU.
        // The exponential phases of the two Q tiles' warps that share this SM sub-partition
        // (warps w and w + 4) alternate: tile 0's k-th, tile 1's k-th, tile 0's (k+1)-th, ...,
        // so that each runs with the sub-partition's MUFU to itself.
        if (t == 1 || kx > 0) {
          ok = bounded_wait(go(t, wq), (t == 0 ? kx - 1 : kx) & 1u, ctl);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
        uint64_t negm2 = ptx::f2x(-m_run, -m_run);
        asm volatile("" : "+l"(negm2)::"memory");  // the exponentials below follow the wait
        const uint64_t sl2x2 = ptx::f2x(sl2, sl2);
        uint64_t lacc0 = 0, lacc1 = 0;  // packed row sums (0 bits == +0.0f)
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const uint64_t x2 = ptx::fma2(ptx::f2x(u2f(sr[2 * c]), u2f(sr[2 * c + 1])), sl2x2, negm2);
          float p0, p1;
          if (emulated_pair(c)) {
            exp2_fma_pair(x2, p0, p1);
          } else {
            float x0, x1;
            ptx::f2x_split(x2, x0, x1);
            p0 = ptx::ex2(x0);
            p1 = ptx::ex2(x1);
          }
          pk[c] = ptx::pack_bf16(p0, p1);
          // Row sum of the bf16-rounded probabilities, i.e. of exactly the weights P V uses.
          if (c & 1)
            madd2(lacc1, pk[c]);
          else
            madd2(lacc0, pk[c]);
        }
        {
          float a0, a1, b0, b1;
          ptx::f2x_split(lacc0, a0, a1);
          ptx::f2x_split(lacc1, b0, b1);
          l_run += (a0 + a1) + (b0 + b1);
        }
        asm volatile("" ::"f"(l_run) : "memory");  // every exponential is done before the hand-over
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(go(1 - t, wq));
        ++kx;
        // P_t and O_t are those of the previous P V of this tile until it completes.
        if (npv > 0) {
          ok = bounded_wait(p_free(t), (npv - 1) & 1u, ctl);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ptx::tc_fence_after();
        }
        if (__any_sync(0xffffffffu, rescale)) {
          const float a = rescale ? alpha : 1.f;
#pragma unroll 1
          for (int cc = 0; cc < DCH * 4; ++cc) {
            uint32_t o[16];
            ptx::tmem_ld16(tO + cc * 16, o);
            ptx::tmem_wait_ld();
            ptx::reg_fence16(o);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(u2f(o[i]) * a);
            ptx::tmem_st16(tO + cc * 16, o);
          }
          ptx::tmem_wait_st();
        }
        // The row of P into shared memory: chunk c (keys 8c .. 8c+7) of panel c / 8 lands at
        // 16-byte column (c % 8) ^ (row % 8).
#pragma unroll
        for (int c = 0; c < 16; ++c)
          ptx::st_shared_v4(p_row + static_cast<uint32_t>(c >> 3) * kChunkBytes +
                                ((static_cast<uint32_t>(c & 7) ^ p_sw) << 4),
                            pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(p_full(t));  // one arrival per warp
        ++npv;
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      ok = bounded_wait(p_free(t), (npv - 1) & 1u, ctl);  // the item's last P V
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      // Store-issue span of this warp's share of the tile (kSeqScatterSpans): SM clock before
      // its first store is prepared and after its last store is issued, and the global timer.
      [[maybe_unused]] unsigned long long span_clk0 = 0, span_ns0 = 0;
      if constexpr (EPI == kSeqScatterSpans) {
        span_clk0 = clock64();
        span_ns0 = ptx::globaltimer();
      }
      const float inv_l = 1.f / l_run;
      // Destination of this thread's row.
      const int s_row = q0 + 128 * t + row;
      uint8_t *dst_row = nullptr;
      if (s_row < p.S) {
        if constexpr (EPI == kSeqScatter || EPI == kSeqScatterSpans) {
          const int b = bh / p.H;
          const int h = bh - b * p.H + p.head_offset;  // global head index
          const int r = s_row / p.S_local;
          const int sl = s_row - r * p.S_local;
          dst_row = static_cast<uint8_t *>(p.dest[r]) +
                    ((static_cast<size_t>(b) * p.S_local + sl) * p.H_dest + h) * static_cast<size_t>(D) * 2;
        } else {
          constexpr size_t kOutBytes = EPI == kPartial ? 4 : 2;
          dst_row = static_cast<uint8_t *>(p.out) +
                    (static_cast<size_t>(bh) * p.S + s_row) * static_cast<size_t>(D) * kOutBytes;
        }
        if constexpr (EPI == kPartial) {
          // log sum_j exp(scale * s_j) = ln 2 * (m + log2 l), m and l in the exp2 domain
          // (l sums the same bf16-rounded weights that P V used).
          p.lse[static_cast<size_t>(bh) * p.S + s_row] = (m_run + log2f(l_run)) * 0.69314718055994531f;
        }
      }
      if constexpr (EPI == kSeqScatter || EPI == kSeqScatterSpans) {
        // Exchange epilogue: each thread writes its own row straight from the TMEM load, in
        // order along the row: 32 bytes at a time where the row starts on a 32-byte boundary
        // (each lane then writes whole L2 sectors), else 16.  No staging in shared memory:
        // while the next item's Q K^T MMAs read both operands from shared memory, staged
        // stores took several times longer to issue (per-tile store-issue span 5.5 us staged,
        // 3.9 us direct with 16-byte stores, 2.5 us with 32-byte ones).  The stores are not
        // waited for: the warp goes straight on to its next tile while they drain.
        constexpr int kEB = EPI == kPartial ? 4 : 2;        // bytes per output element
        constexpr int kChunksPerLd = 2 * kEB;                // 16-byte chunks per 32 columns
        const int nch = D * kEB / 16;                        // 16-byte chunks per output row
        // whole 32-byte pairs of chunks: the row starts on a 32-byte boundary and has an even
        // number of chunks (bf16 rows only)
        const bool row32 = kEB == 2 && (nch & 1) == 0 &&
                           (reinterpret_cast<uintptr_t>(dst_row) & 31u) == 0;
        // The epilogue loops are not unrolled: they run once per work item, and the smaller
        // kernel body measured 0.5-4% faster over the workloads (the difference is in the
        // compiled key loop, not in the epilogue itself).
#pragma unroll 1
        for (int cc = 0; cc < DCH * 2; ++cc) {
          uint32_t o[32];
          ptx::tmem_ld32(tO + cc * 32, o);
          ptx::tmem_wait_ld();
          ptx::reg_fence32(o);
          if (dst_row != nullptr && row32) {
            // 32-byte stores: every lane writes whole L2 sectors of its row
#pragma unroll
            for (int q8 = 0; q8 < kChunksPerLd / 2; ++q8) {
              const int c = cc * kChunksPerLd + 2 * q8;  // first 16-byte chunk of the pair
              if (c < nch) {
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  w[i] = ptx::pack_bf16(u2f(o[16 * q8 + 2 * i]) * inv_l, u2f(o[16 * q8 + 2 * i + 1]) * inv_l);
                ptx::st_global_v8(dst_row + c * 16, w);
              }
            }
          } else if (dst_row != nullptr) {
#pragma unroll
            for (int q4 = 0; q4 < kChunksPerLd; ++q4) {
              const int c = cc * kChunksPerLd + q4;  // 16-byte chunk of the output row
              if (c < nch) {
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  if constexpr (kEB == 2)
                    w[i] = ptx::pack_bf16(u2f(o[8 * q4 + 2 * i]) * inv_l, u2f(o[8 * q4 + 2 * i + 1]) * inv_l);
                  else
                    w[i] = f2u(u2f(o[4 * q4 + i]) * inv_l);
                }
                ptx::st_global_v4(dst_row + c * 16, make_uint4(w[0], w[1], w[2], w[3]));
              }
            }
          }
        }
        if (p.slab_flags[0] != nullptr) {
          // Arrival counters: after the warp's stores (ordered before the leader's release by
          // the warp barrier), one lane per destination slab among the warp's 32 rows adds
          // that slab's row count with a system-scope release.  The release waits for the
          // warp's stores to become visible, so this path costs the storing warps that wait;
          // without counters the stores are never waited for.
          const int r = dst_row != nullptr ? s_row / p.S_local : -1;
          __syncwarp();
          unsigned pending = __ballot_sync(0xffffffffu, r >= 0);
          while (pending != 0u) {
            const int leader = __ffs(pending) - 1;
            const int rl = __shfl_sync(0xffffffffu, r, leader);
            const unsigned same = __ballot_sync(0xffffffffu, r == rl);
            if (lane == leader) ptx::red_release_sys_add(p.slab_flags[rl], __popc(same));
            pending &= ~same;
          }
        }
      } else {
        // Head-major and partial epilogues: rounds of kRows rows per warp (16 in bf16, 8 in
        // fp32) staged in shared memory (chunk order rotated by row to spread banks), then
        // whole rows written with consecutive lanes on consecutive 16-byte chunks (storing
        // each thread's row directly made the L2 read the partly written sectors of these
        // contiguous rows back from DRAM: +1.1 bytes read per byte written).  The stores are not waited for: the warp goes
        // straight on to its next tile while they drain.
        // O is read from TMEM once per round, 32 columns at a time (the warp-collective load
        // brings all 32 rows; the lanes of the current round keep theirs).
        constexpr int kEB = EPI == kPartial ? 4 : 2;        // bytes per output element
        constexpr int kRows = kStageRows * 2 / kEB;          // rows per round
        constexpr int kRowBytes = L::kStageRowBytes * kEB / 2;
        constexpr int kChunksPerLd = 2 * kEB;                // 16-byte chunks per 32 columns
        const int nch = D * kEB / 16;                        // 16-byte chunks per output row
#pragma unroll 1
        for (int rd = 0; rd < 32 / kRows; ++rd) {
          const bool mine = lane / kRows == rd;
          const int rr = lane % kRows;
          const int rot = rr % nch;
          uint8_t *my = stg + rr * kRowBytes;
#pragma unroll 1
          for (int cc = 0; cc < DCH * 2; ++cc) {
            uint32_t o[32];
            ptx::tmem_ld32(tO + cc * 32, o);
            ptx::tmem_wait_ld();
            ptx::reg_fence32(o);
            if (mine) {
#pragma unroll
              for (int q4 = 0; q4 < kChunksPerLd; ++q4) {
                const int c = cc * kChunksPerLd + q4;  // 16-byte chunk of the output row
                if (c < nch) {
                  int pc = c + rot;
                  if (pc >= nch) pc -= nch;
                  uint32_t w[4];
#pragma unroll
                  for (int i = 0; i < 4; ++i) {
                    if constexpr (kEB == 2)
                      w[i] = ptx::pack_bf16(u2f(o[8 * q4 + 2 * i]) * inv_l, u2f(o[8 * q4 + 2 * i + 1]) * inv_l);
                    else
                      w[i] = f2u(u2f(o[4 * q4 + i]) * inv_l);
                  }
                  *reinterpret_cast<uint4 *>(my + pc * 16) = make_uint4(w[0], w[1], w[2], w[3]);
                }
              }
            }
          }
          if (mine) rowptr[rr] = dst_row;
          __syncwarp();
          for (int idx = lane; idx < kRows * nch; idx += 32) {
            const int r2 = idx / nch;
            const int c = idx - r2 * nch;
            uint8_t *dr = rowptr[r2];
            if (dr != nullptr) {
              int pc = c + r2 % nch;
              if (pc >= nch) pc -= nch;
              const uint4 v = *reinterpret_cast<const uint4 *>(stg + r2 * kRowBytes + pc * 16);
              ptx::st_global_v4(dr + c * 16, v);
            }
          }
          __syncwarp();
        }
      }
      if constexpr (EPI == kSeqScatterSpans) {
        // The stores above are only issued, not complete: this is the sender-visible time.
        const unsigned long long clk1 = clock64();
        if (lane == 0) {
          unsigned long long *sp = p.spans + ((static_cast<size_t>(item) * 2 + t) * 4 + wq) * 3;
          sp[0] = span_clk0;
          sp[1] = clk1;
          sp[2] = span_ns0;
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

template <int DCH, int EPI, int KSQ = DCH * 4>
cudaError_t launch_impl(const AttnParams &p, cudaStream_t stream) {
  using L = Smem<DCH>;
  static_assert(L::kAlloc <= 232448, "shared memory budget exceeded");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  constexpr int kMaxDevices = 64;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  // Per device, once (threads racing on a first call wait for the one that sets it up): the
  // opt-in to the dynamic shared memory this instance needs.
  static std::once_flag once[kMaxDevices];
  static cudaError_t setup[kMaxDevices];
  std::call_once(once[dev], [dev] {
    setup[dev] = cudaFuncSetAttribute(attn_fwd_kernel<DCH, EPI, KSQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(L::kAlloc));
  });
  if (setup[dev] != cudaSuccess) return setup[dev];
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int grid = p.n_items < sms ? p.n_items : sms;
  attn_fwd_kernel<DCH, EPI, KSQ><<<grid, kThreads, L::kAlloc, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t attention_smem_bytes(int dch) { return dch == 1 ? Smem<1>::kAlloc : Smem<2>::kAlloc; }

cudaError_t launch_attention(const AttnParams &p, int epilogue, cudaStream_t stream) {
  const int dch = p.D <= 64 ? 1 : 2;
  if (epilogue == kSeqScatterSpans)
    return dch == 1 ? launch_impl<1, kSeqScatterSpans>(p, stream) : launch_impl<2, kSeqScatterSpans>(p, stream);
  if (dch == 1)
    return epilogue == kHeadMajor  ? launch_impl<1, kHeadMajor>(p, stream)
           : epilogue == kPartial ? launch_impl<1, kPartial>(p, stream)
                                  : launch_impl<1, kSeqScatter>(p, stream);
  if (p.D <= 80)  // 5 K steps of Q K^T carry the head dimension (the last one partly zero fill)
    return epilogue == kHeadMajor  ? launch_impl<2, kHeadMajor, 5>(p, stream)
           : epilogue == kPartial ? launch_impl<2, kPartial, 5>(p, stream)
                                  : launch_impl<2, kSeqScatter, 5>(p, stream);
  return epilogue == kHeadMajor  ? launch_impl<2, kHeadMajor>(p, stream)
         : epilogue == kPartial ? launch_impl<2, kPartial>(p, stream)
                                : launch_impl<2, kSeqScatter>(p, stream);
}

}  // namespace xs
