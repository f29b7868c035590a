// BLASST skip-softmax attention for B200 (sm_100a): forward with tile
// skipping and the multi-threshold calibration pass.
//
// One CTA takes two consecutive 128-row query blocks (X = A, B) of one
// (sequence, head) and walks the sequence's KV tiles in order; both query
// blocks share every K and V tile staged in shared memory. Warp roles:
//   warps 0-3 / 4-7  softmax of query block A / B, one query row per thread:
//           row max of S_X in the log2 domain, the block's skip vote
//           d_j < log2(lambda) (Model-Optimizer commit page, "Triton kernels":
//           tiles whose max score is far below the running max are skipped,
//           no V load, softmax or accumulation), exponentials against a lazily
//           rescaled reference max, P_X (bf16) written over S_X in TMEM, and
//           the epilogue O_X / l -> bf16;
//   warp 8  TMA producer: Q_A and Q_B once, K tiles through a 3-stage ring and
//           V tiles through a 2-stage ring -- V_j only once A or B has decided
//           to keep tile j (a tile both skip issues no V load);
//   warp 9  tcgen05 issuer, per KV tile j and per block X in order A, B:
//           O_X += P_X V_j (when X keeps j, P_X read from TMEM), then
//           S_X = Q_X K_{j+1}^T into the same TMEM columns (bf16 operands, or
//           E4M3 ones with per-tensor descales folded into the score scale;
//           with E4M3 V the P V product runs on E4M3 P and V as well).
// tcgen05 MMAs issued by one thread execute in issue order, so the S MMA
// cannot overwrite P_X before the PV MMA ahead of it has read P_X; and a
// commit tracks every earlier MMA of the thread, so when S_X(j+1) is reported
// complete every MMA into O_X issued before it has completed too (the softmax
// may rescale O_X and overwrite the P_X columns without a further wait).
// A block's skip decision reaches the issuer as a tagged word in shared
// memory that it polls with acquire loads (on the issuing thread a barrier
// wait stalls longer behind its in-flight MMAs than a load does); the
// producer, which decides the V loads, polls the same word with a back-off.
// In the skipping kernel the decision also says that K_{j+1} has landed (the
// group's first warp waits for it before it reads S_X(j)), so the issuer puts
// S_X(j+1) in flight with no wait of its own.
// The two softmax groups run out of phase: one group's exponentials overlap
// the MMAs of the other.
// TMEM (512 columns): S_A [0,128) S_B [128,256) O_A [256,256+D)
// O_B [384,384+D); P_X is written over S_X as packed bf16 pairs, kv [0,64) to
// columns [0,32) and kv [64,128) to [64,96) (E4M3 P, four kv per column, to
// [0,16) and [64,80)): the upper half is stored as soon as it is computed
// (its S columns have been read) while the lower half of S is still being
// read back, and the issuer starts O_X += P_X V on that half while the softmax
// exponentiates the other one.
//
// Every wait on an mbarrier is bounded in time; when one runs out the CTA
// records SSA_ERR_TIMEOUT in the device status word, the other roles see the
// abort flag at their next wait, in-flight TMA loads and MMAs are drained
// (again with a bound) and TMEM is released before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <initializer_list>

#include "sm100.cuh"
#include "ssa.h"

namespace ssa {
namespace {

using namespace sm100;

constexpr int kBM = SSA_TILE;  // query rows per block
constexpr int kBN = SSA_TILE;  // key/value rows per tile
constexpr int kQBlocks = 2;    // query blocks per CTA
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kCalWindow = 16;  // calibration: tiles whose votes are counted together
constexpr int kDecRing = 4;  // > kKStages - 1: bounds how far a vote runs ahead of its readers
constexpr uint32_t kTmemCols = 512;
__host__ __device__ constexpr uint32_t col_S(int x) { return x ? 128u : 0u; }    // S_X (and P_X)
__host__ __device__ constexpr uint32_t col_O(int x) { return x ? 384u : 256u; }  // O_X
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 256 before a rescale
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kStatusTimeout = 1;
constexpr int kStatusDeviceArg = 2;
constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr int kVoteBarrier = 1;  // named barriers 1 and 2: the vote of softmax group A and B

enum Mode : int { kDense = 0, kSkip = 1, kCalib = 2 };

__device__ int g_status;  // sticky error bits of this device, read by ssa_get_error
thread_local const char* t_last_cuda_error = "no error";

int cuda_fail(cudaError_t e) {
  t_last_cuda_error = cudaGetErrorString(e);
  return SSA_ERR_CUDA;
}

struct Params {
  const int32_t* cu_seqlens;
  __nv_bfloat16* out;
  int32_t* skip_counter;
  int32_t* counts;
  uint32_t* bitmap;
  float* tile_stat;
  int batch, total_tokens, num_heads, max_tiles, bitmap_words;
  int nq_check;  // q-blocks the per-unit outputs are sized for, or -1 when there are none
  float c;    // fp32(softmax_scale * log2 e)
  float v_scale;  // multiplies the output: the V descale for E4M3 V, else 1
  float tsf;  // threshold_scale_factor (kSkip)
  int n_cal;
  float Lcal[SSA_MAX_THRESHOLDS];  // fp32(log2 lambda_k) (kCalib)
};

struct Ctl {
  uint64_t bar_q;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[kQBlocks], p_hi[kQBlocks], p_ready[kQBlocks];
  uint64_t o_final, drain;
  uint32_t tmem_base;
  int abort_flag;
  int dec[kQBlocks][kDecRing];  // decision of tile j in slot j % kDecRing: ((j + 1) << 1) | skip
  float red[kQBlocks][2][4];
  float cal_red[kQBlocks][2][kCalWindow][4];  // calibration: each warp's vote per tile, double-buffered windows
  int seq, qb_a, has_b, S, start, gqb_a, nq_total;
};

// Operand precisions: bf16 everywhere; E4M3 Q and K; E4M3 Q, K, V and P.
enum Prec : int { kBf16 = 0, kQK8 = 1, kQKV8 = 2 };

// Shared-memory layout. Q and K are bf16, or E4M3 bytes from kQK8 on; V is
// bf16, or E4M3 bytes for kQKV8. Every tile is stored as chunks of 128 rows x
// 128 B with the 128-byte swizzle.
template <int D, int PREC>
struct Layout {
  static constexpr int kQKElem = PREC >= kQK8 ? 1 : 2;        // bytes per Q/K element
  static constexpr int kQKTileBytes = kBM * D * kQKElem;
  static constexpr int kQKChunkElems = 128 / kQKElem;         // Q/K elements per 128-B row of a chunk
  static constexpr int kQKChunks = D / kQKChunkElems;
  static constexpr int kVElem = PREC == kQKV8 ? 1 : 2;        // bytes per V element
  static constexpr int kVChunkElems = 128 / kVElem;           // V elements per 128-B row of a chunk
  static constexpr int kVChunks = D / kVChunkElems;
  static constexpr int kVTileBytes = kBN * D * kVElem;
  static constexpr int kChunkBytes = kBM * 128;
  static constexpr int kQ = 0;  // Q_A, then Q_B
  static constexpr int kK = kQ + kQBlocks * kQKTileBytes;
  static constexpr int kV = kK + kKStages * kQKTileBytes;
  static constexpr int kCtl = kV + kVStages * kVTileBytes;
  static constexpr int kBytes = kCtl + static_cast<int>(sizeof(Ctl));
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 B (128B swizzle atoms)
  static_assert(kAlloc <= 232448, "shared memory beyond the 227 KB a CTA may use");
};

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        atomicOr(&g_status, kStatusTimeout);
        return false;
      }
    }
  }
}

// Bounded poll of a tagged decision word until it carries `tag` (the tile
// index + 1); returns the word. Same limit and abort protocol as wait_bar.
__device__ __forceinline__ bool wait_decision(uint32_t addr, int tag, int& word, volatile int* abort_flag) {
  word = ld_acquire_shared(addr);
  if ((word >> 1) == tag) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    word = ld_acquire_shared(addr);
    if ((word >> 1) == tag) return true;
    if ((i & 31u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        atomicOr(&g_status, kStatusTimeout);
        return false;
      }
    }
  }
}

// Same, for a waiter that is in no hurry: sleeps between polls, so that it
// leaves shared-memory bandwidth to the tensor cores' operand reads.
__device__ __forceinline__ bool wait_decision_sleep(uint32_t addr, int tag, int& word, volatile int* abort_flag) {
  word = ld_acquire_shared(addr);
  if ((word >> 1) == tag) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    __nanosleep(64);
    word = ld_acquire_shared(addr);
    if ((word >> 1) == tag) return true;
    if ((i & 15u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        atomicOr(&g_status, kStatusTimeout);
        return false;
      }
    }
  }
}

// One arrival for the whole warp: order this warp's finished tcgen05 loads
// and stores before the thread synchronisation, gather the warp, and let
// lane 0 arrive (one atomic on the barrier word instead of 32).
__device__ __forceinline__ void warp_arrive(uint32_t bar, int lane) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// Warp-uniform bounded wait: every lane returns the same verdict.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  return __all_sync(kFull, wait_bar(bar, parity, abort_flag));
}

// Wait that ignores the abort flag (used to drain in-flight async work).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_status, kStatusTimeout);
      return;
    }
  }
}

// Maps this CTA (blockIdx.x) to its (sequence, pair of query blocks) and
// validates cu_seqlens; run by the whole of warp 0. For batches of up to 32
// sequences the pairs are numbered longest sequence first (ties by index), so
// the units with the longest KV walks start first and short ones fill the end
// of the grid; larger batches keep sequence order. Either way the per-unit
// outputs are indexed by the global q-block in sequence order. A CTA past the
// last pair gets ctl.seq = -1, and so does every CTA when the input is
// inconsistent: cu_seqlens negative, decreasing or past total_tokens, a
// sequence longer than max_seqlen where the diagnostics are sized from it, or
// a q-block count other than the one the caller sized its per-unit outputs
// for (p.nq_check >= 0). Inconsistencies are reported in the status word.
__device__ void locate_unit(const Params& p, bool need_max, int lane, Ctl& ctl) {
  const int x = static_cast<int>(blockIdx.x);
  int seq = -1, qb_a = 0, has_b = 0, start = 0, S = 0, gqb_a = 0, bad = 0, nq_total = 0;
  if (p.batch <= 32) {
    const int b = lane;  // one sequence per lane
    int lo = 0, len = 0, nq = 0, np = 0;
    if (b < p.batch) {
      lo = p.cu_seqlens[b];
      const int hi = p.cu_seqlens[b + 1];
      len = hi - lo;
      if (lo < 0 || len < 0 || hi > p.total_tokens) bad = 1;
      nq = (len + kBM - 1) / kBM;
      np = (nq + 1) / 2;
      if (need_max && nq > p.max_tiles) bad = 1;
    }
    bad = __any_sync(kFull, bad) ? 1 : 0;
    int q_off = nq;  // inclusive prefix sum of q-blocks in sequence order
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(kFull, q_off, o);
      if (lane >= o) q_off += t;
    }
    nq_total = __shfl_sync(kFull, q_off, 31);
    q_off -= nq;
    int p_off = 0;  // first pair of sequence b in longest-first order
    for (int o = 0; o < p.batch; ++o) {
      const int len_o = __shfl_sync(kFull, len, o), np_o = __shfl_sync(kFull, np, o);
      if (len_o > len || (len_o == len && o < b)) p_off += np_o;
    }
    const unsigned who = __ballot_sync(kFull, b < p.batch && x >= p_off && x < p_off + np);
    if (who) {
      const int src = __ffs(static_cast<int>(who)) - 1;
      const int pair = __shfl_sync(kFull, x - p_off, src);
      const int nq_s = __shfl_sync(kFull, nq, src);
      seq = src;
      qb_a = 2 * pair;
      has_b = qb_a + 1 < nq_s ? 1 : 0;
      gqb_a = __shfl_sync(kFull, q_off, src) + qb_a;
      start = __shfl_sync(kFull, lo, src);
      S = __shfl_sync(kFull, len, src);
    }
  } else if (lane == 0) {
    int accp = 0;
    int prev = p.cu_seqlens[0];
    if (prev < 0) bad = 1;
    for (int b = 0; b < p.batch && !bad; ++b) {
      const int nxt = p.cu_seqlens[b + 1];
      const int len = nxt - prev;
      if (len < 0 || nxt > p.total_tokens) {
        bad = 1;
        break;
      }
      const int nq = (len + kBM - 1) / kBM;
      const int np = (nq + 1) / 2;
      if (need_max && nq > p.max_tiles) bad = 1;
      if (seq < 0 && x < accp + np) {
        seq = b;
        qb_a = 2 * (x - accp);
        has_b = qb_a + 1 < nq ? 1 : 0;
        gqb_a = nq_total + qb_a;
        start = prev;
        S = len;
      }
      nq_total += nq;
      accp += np;
      prev = nxt;
    }
  }
  if (lane == 0) {
    if (!bad && p.nq_check >= 0 && nq_total != p.nq_check) bad = 1;
    if (bad) {
      if (x == 0) atomicOr(&g_status, kStatusDeviceArg);
      seq = -1;
    }
    ctl.seq = seq;
    ctl.qb_a = qb_a;
    ctl.has_b = has_b;
    ctl.S = S;
    ctl.start = start;
    ctl.gqb_a = gqb_a;
    ctl.nq_total = nq_total;
  }
}

template <int D, int MODE, bool EX, int PREC>
__global__ void __launch_bounds__(kThreads, 1)
    ssa_attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ Params p) {
  using L = Layout<D, PREC>;
  constexpr bool F8 = PREC >= kQK8;    // S = Q K^T on E4M3 operands
  constexpr bool F8V = PREC == kQKV8;  // O += P V on E4M3 operands as well
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + L::kCtl);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;

  if (warp == 0) locate_unit(p, EX, lane, ctl);
  __syncthreads();
  if (ctl.seq < 0) return;  // uniform: no unit for this CTA (or bad input)

  const int qb_a = ctl.qb_a, S = ctl.S, seq_start = ctl.start;
  const int nx = ctl.has_b ? 2 : 1;  // query blocks this CTA holds
  const int nkv = (S + kBN - 1) / kBN;
  volatile int* abort_flag = &ctl.abort_flag;

  const uint32_t bar_q = smem_u32(&ctl.bar_q);
  auto k_full = [&](int i) { return smem_u32(&ctl.k_full[i]); };
  auto k_empty = [&](int i) { return smem_u32(&ctl.k_empty[i]); };
  auto v_full = [&](int i) { return smem_u32(&ctl.v_full[i]); };
  auto v_empty = [&](int i) { return smem_u32(&ctl.v_empty[i]); };
  auto s_full = [&](int x) { return smem_u32(&ctl.s_full[x]); };
  auto p_ready = [&](int x) { return smem_u32(&ctl.p_ready[x]); };
  auto p_hi = [&](int x) { return smem_u32(&ctl.p_hi[x]); };
  const uint32_t o_final = smem_u32(&ctl.o_final);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(v_full(i), 1);
      mbar_init(v_empty(i), 1);
    }
    for (int x = 0; x < kQBlocks; ++x) {
      mbar_init(s_full(x), 1);
      mbar_init(p_ready(x), 4);  // one arrival per softmax warp of the group, per kept tile
      mbar_init(p_hi(x), 4);     // the same, once the upper half of P_X is stored
    }
    mbar_init(o_final, 1);
    mbar_init(smem_u32(&ctl.drain), 1);
    ctl.abort_flag = 0;
    for (int x = 0; x < kQBlocks; ++x)
      for (int i = 0; i < kDecRing; ++i) ctl.dec[x][i] = 0;  // tag 0: no tile yet
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&ctl.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(bar_q, nx * L::kQKTileBytes);
      for (int x = 0; x < nx; ++x) {
        const uint32_t q_s = smem_u32(smem + L::kQ + x * L::kQKTileBytes);
        for (int ch = 0; ch < L::kQKChunks; ++ch)
          tma_load_3d(q_s + ch * L::kChunkBytes, &tmQ, bar_q, ch * L::kQKChunkElems, head,
                      seq_start + (qb_a + x) * kBM);
      }
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (int j = 0; j < nkv && ok; ++j) {
        for (; k_issued < nkv && k_issued < j + kKStages; ++k_issued) {
          const int st = k_issued % kKStages;
          if (k_issued >= kKStages && !wait_bar(k_empty(st), ((k_issued / kKStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(smem + L::kK + st * L::kQKTileBytes);
          mbar_arrive_expect_tx(k_full(st), L::kQKTileBytes);
          for (int ch = 0; ch < L::kQKChunks; ++ch)
            tma_load_3d(dst + ch * L::kChunkBytes, &tmK, k_full(st), ch * L::kQKChunkElems, head,
                        seq_start + k_issued * kBN);
        }
        if (!ok) break;
        bool need_v = true;
        if (MODE == kSkip) {  // V_j is needed when either block keeps tile j
          need_v = false;
          for (int x = 0; x < nx && !need_v; ++x) {
            int word;
            if (!wait_decision_sleep(smem_u32(&ctl.dec[x][j % kDecRing]), j + 1, word, abort_flag)) {
              ok = false;
              break;
            }
            need_v = (word & 1) == 0;
          }
          if (!ok) break;
        }
        if (need_v) {
          const int vs = v_issued % kVStages;
          if (v_issued >= kVStages && !wait_bar(v_empty(vs), ((v_issued / kVStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(smem + L::kV + vs * L::kVTileBytes);
          mbar_arrive_expect_tx(v_full(vs), L::kVTileBytes);
          for (int ch = 0; ch < L::kVChunks; ++ch)
            tma_load_3d(dst + ch * L::kChunkBytes, &tmV, v_full(vs), ch * L::kVChunkElems, head,
                        seq_start + j * kBN);
          ++v_issued;
        }
      }
      if (!ok) {  // drain the loads still in flight before shared memory goes away
        drain_wait(bar_q, 0);
        for (int st = 0; st < kKStages; ++st)
          if (k_issued > st) drain_wait(k_full(st), ((k_issued - 1 - st) / kKStages) & 1);
        for (int st = 0; st < kVStages; ++st)
          if (v_issued > st) drain_wait(v_full(st), ((v_issued - 1 - st) / kVStages) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------- tcgen05 issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = F8 ? idesc_e4m3_f32(kBM, kBN) : idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idesc_pv = F8V ? idesc_e4m3_f32(kBM, D, true) : idesc_bf16_f32(kBM, D, true);
      // S_X = Q_X K_t^T (the caller has made sure K_t has landed and that
      // nothing still needs S_X's previous contents).
      auto issue_qk = [&](int x, int t) {
        const uint32_t q_s = smem_u32(smem + L::kQ + x * L::kQKTileBytes);
        const uint32_t k_s = smem_u32(smem + L::kK + (t % kKStages) * L::kQKTileBytes);
        const uint32_t d_tmem = tmem + col_S(x);
        // Shared-memory addresses stay below 256 KB, so the 14-bit address
        // field of a descriptor takes an offset by plain addition: each MMA's
        // descriptors are the tile's plus a constant, added to the low word
        // alone (it cannot carry out of the field), which keeps the single
        // issuing thread, on the critical path of every tile, short.
        const uint64_t da0 = smem_desc_sw128(q_s, 16, 1024), db0 = smem_desc_sw128(k_s, 16, 1024);
        const uint32_t a_lo = static_cast<uint32_t>(da0), b_lo = static_cast<uint32_t>(db0);
        const uint64_t a_hi = da0 & 0xFFFFFFFF00000000ull, b_hi = db0 & 0xFFFFFFFF00000000ull;
#pragma unroll
        for (int ks = 0; ks < D * L::kQKElem / 32; ++ks) {
          // K-major, 128B swizzle: each MMA takes 32 B of K (16 bf16 or 32
          // E4M3 elements), 32 B apart inside a 128-B row; every 128 B of a
          // row start a new 16 KB chunk.
          const uint32_t off = (ks >> 2) * L::kChunkBytes + (ks & 3) * 32;
          const uint64_t da = a_hi | (a_lo + (off >> 4)), db = b_hi | (b_lo + (off >> 4));
          if (F8)
            mma_ss_f8(d_tmem, da, db, idesc_qk, ks > 0 ? 1u : 0u);
          else
            mma_ss(d_tmem, da, db, idesc_qk, ks > 0 ? 1u : 0u);
        }
        tc_commit(s_full(x));
      };
      // Half `half` of O_X += P_X V_vs from the TMEM copy of P_X: half 1 (kv
      // [64,128)) is issued as soon as that half of P_X is stored, while the
      // softmax still exponentiates the lower half; half 0 (kv [0,64)) once
      // all of P_X is in place. P_X sits at columns [0,32) and [64,96) of S_X
      // as bf16 pairs, or at [0,16) and [64,80) as E4M3.
      auto issue_pv = [&](int x, int vs, int half, bool accumulate) {
        const uint32_t p_tmem = tmem + col_S(x);
        const uint32_t v_s = smem_u32(smem + L::kV + vs * L::kVTileBytes);
        if (F8V) {
          // E4M3 P four to a column, 32 kv per instruction; V MN-major with
          // its 128 E4M3 d values in one 128-B row per kv: 32 rows = 4 KB per
          // k step, one swizzle atom across d (LBO unused), 8-row groups 1 KB
          // apart.
          const uint64_t vd0 = smem_desc_sw128(v_s, 0, 1024);
          const uint32_t v_lo = static_cast<uint32_t>(vd0);
          const uint64_t v_hi = vd0 & 0xFFFFFFFF00000000ull;
#pragma unroll
          for (int i = 0; i < kBN / 64; ++i) {
            const int ks = half * (kBN / 64) + i;
            const uint32_t p_col = ks * 8 + (half ? 48 : 0);
            mma_ts_f8(tmem + col_O(x), p_tmem + p_col, v_hi | (v_lo + static_cast<uint32_t>(ks * 32 * 128 >> 4)),
                      idesc_pv, (accumulate || i > 0) ? 1u : 0u);
          }
        } else {
          // V is MN-major (d contiguous): 16 kv rows = 2 KB per k step; the
          // second 64-column chunk of d sits one 16 KB chunk further (LBO).
          const uint64_t vd0 = smem_desc_sw128(v_s, L::kChunkBytes, 1024);
          const uint32_t v_lo = static_cast<uint32_t>(vd0);
          const uint64_t v_hi = vd0 & 0xFFFFFFFF00000000ull;
#pragma unroll
          for (int i = 0; i < kBN / 32; ++i) {
            const int ks = half * (kBN / 32) + i;
            const uint32_t p_col = ks * 8 + (half ? 32 : 0);
            mma_ts(tmem + col_O(x), p_tmem + p_col, v_hi | (v_lo + static_cast<uint32_t>(ks * 16 * 128 >> 4)),
                   idesc_pv, (accumulate || i > 0) ? 1u : 0u);
          }
        }
      };
      bool ok = wait_bar(bar_q, 0, abort_flag) && wait_bar(k_full(0), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int x = 0; x < nx; ++x) issue_qk(x, 0);
        tc_commit(k_empty(0));
      }
      int kept[kQBlocks] = {0, 0};
      int v_used = 0;
      for (int j = 0; ok && j < nkv; ++j) {
        const int t = j + 1;  // S_X(t) is issued right behind O_X += P_X(j) V_j
        // Waits that are normally already satisfied (K_{j+1} and V_j in the
        // dense and calibration orders) come first, while no MMA of this tile
        // is in flight: a wait behind in-flight MMAs stalls the issuer. In the
        // skipping order the decisions polled below imply K_{j+1}.
        if (MODE != kSkip && t < nkv && !(ok = wait_bar(k_full(t % kKStages), (t / kKStages) & 1, abort_flag)))
          break;
        bool v_waited = false;
        if (MODE != kSkip) {
          if (!(ok = wait_bar(v_full(v_used % kVStages), (v_used / kVStages) & 1, abort_flag))) break;
          v_waited = true;
        }
        for (int x = 0; x < nx; ++x) {
          bool skip = false;
          if (MODE == kSkip) {
            // The decision also says every warp of the group has read S_X(j)
            // and that K_{j+1} has landed.
            int word;
            if (!(ok = wait_decision(smem_u32(&ctl.dec[x][j % kDecRing]), j + 1, word, abort_flag))) break;
            skip = (word & 1) != 0;
          }
          if (!skip) {
            if (!(ok = wait_bar(p_hi(x), kept[x] & 1, abort_flag))) break;
            if (!v_waited) {
              if (!(ok = wait_bar(v_full(v_used % kVStages), (v_used / kVStages) & 1, abort_flag))) break;
              v_waited = true;
            }
            tc_fence_after();
            issue_pv(x, v_used % kVStages, 1, kept[x] > 0);
            if (!(ok = wait_bar(p_ready(x), kept[x] & 1, abort_flag))) break;
            tc_fence_after();
            issue_pv(x, v_used % kVStages, 0, true);
            ++kept[x];
          }
          if (t < nkv) {
            if (skip) tc_fence_after();  // after a PV the fence above already covers the S MMAs
            issue_qk(x, t);
          }
        }
        if (!ok) break;
        if (v_waited) {  // V_j's stage is free once every PV on it has completed
          tc_commit(v_empty(v_used % kVStages));
          ++v_used;
        }
        if (t < nkv) tc_commit(k_empty(t % kKStages));
      }
      if (ok) {
        tc_commit(o_final);
      } else {  // let every MMA issued so far finish before TMEM is released
        tc_commit(smem_u32(&ctl.drain));
        drain_wait(smem_u32(&ctl.drain), 0);
      }
    }
  } else if (warp < 4 * nx) {
    // ------------------------------------------------------------- softmax
    const int x = warp >> 2;   // query block of this warp's group
    const int wq = warp & 3;   // TMEM lane quadrant = row group inside the block
    const int gt = threadIdx.x & 127;  // thread index inside the group
    const int qb = qb_a + x;
    const int row = wq * 32 + lane;
    const bool row_valid = qb * kBM + row < S;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t col_s = col_S(x), col_o = col_O(x);
    const int vote_bar = kVoteBarrier + x;
    const int64_t unit = static_cast<int64_t>(head) * ctl.nq_total + ctl.gqb_a + x;
    const float c = p.c;
    float Lthr = -INFINITY;
    if (MODE == kSkip) Lthr = static_cast<float>(log2(static_cast<double>(p.tsf) / static_cast<double>(S)));
    float m_true = -INFINITY;  // running max of kept tiles (the skip rule's m_r)
    float m_used = -INFINITY;  // reference max of the exponentials (lags m_true by < kRescaleThreshold)
    float l = 0.f;
    int kept = 0, nskip = 0;
    // Calibration: thread gt counts tile slot (gt & 15) of every window for
    // thresholds (gt >> 4) + 8m, m = 0..3 (up to 32 thresholds).
    int cal_cnt[4] = {0, 0, 0, 0};
    uint32_t bits = 0;
    bool ok = true;

    for (int j = 0; j < nkv; ++j) {
      // Skipping order: the group's first warp (which publishes the decision)
      // makes sure K_{j+1} has landed, while it would wait for S_X(j) anyway.
      if (MODE == kSkip && wq == 0 && j + 1 < nkv &&
          !(ok = warp_wait(k_full((j + 1) % kKStages), ((j + 1) / kKStages) & 1, abort_flag)))
        break;
      if (!(ok = warp_wait(s_full(x), j & 1, abort_flag))) break;
      tc_fence_after();
      // S_X is read whole for the row max; only its upper 64 columns stay in
      // registers, the lower half is read again (asynchronously) for the
      // exponentials of a kept tile, to bound register use.
      const int valid = S - j * kBN;  // valid columns of this tile (masked to -inf past it)
      uint32_t hi[64];
      float mx[8];
      {
        uint32_t sr[128];
        tmem_ld_x128(lane_base + col_s, sr);
        if (valid < kBN) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= valid) sr[i] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = fmaxf(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]));
#pragma unroll
        for (int i = 8; i < 64; ++i)
          mx[i & 7] = fmax3(mx[i & 7], __uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]));
#pragma unroll
        for (int i = 0; i < 64; ++i) hi[i] = sr[64 + i];
      }
      const float tmax = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(fmax3(mx[3], mx[4], mx[5]), mx[6], mx[7])) * c;

      bool skip = false;
      if (MODE == kCalib) {
        // No per-tile barrier: each warp leaves its vote in the current
        // window; once per window (and after the last tile) the group meets
        // and counts every threshold for the window's tiles in parallel.
        const float dr = warp_max_f32(row_valid ? (tmax - m_true) : -INFINITY);
        const int win = j / kCalWindow, slot = j % kCalWindow;
        if (lane == 0) ctl.cal_red[x][win & 1][slot][wq] = dr;
        if (slot == kCalWindow - 1 || j == nkv - 1) {
          named_barrier_sync(vote_bar, 128);
          const int i = gt & (kCalWindow - 1);
          if (i <= slot) {
            volatile float* r = ctl.cal_red[x][win & 1][i];
            const float d = fmaxf(fmaxf(r[0], r[1]), fmaxf(r[2], r[3]));
            if (EX && gt < kCalWindow && p.tile_stat) p.tile_stat[unit * p.max_tiles + win * kCalWindow + i] = d;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const int k = (gt >> 4) + 8 * m;
              if (k < p.n_cal) cal_cnt[m] += d < p.Lcal[k] ? 1 : 0;
            }
          }
        }
      } else if (MODE != kDense || EX) {
        const float dr = warp_max_f32(row_valid ? (tmax - m_true) : -INFINITY);
        if (lane == 0) ctl.red[x][j & 1][wq] = dr;
        // S_X(j) has been read into registers by every warp of the group once
        // this barrier completes: the decision below then also frees S_X.
        tc_fence_before();
        named_barrier_sync(vote_bar, 128);
        volatile float* red = ctl.red[x][j & 1];
        const float d = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
        if (MODE == kSkip) skip = d < Lthr;
        if (EX && gt == 0) {
          if (p.tile_stat) p.tile_stat[unit * p.max_tiles + j] = d;
          bits |= (skip ? 1u : 0u) << (j & 31);
          if ((j & 31) == 31 || j == nkv - 1) {
            if (p.bitmap) p.bitmap[unit * p.bitmap_words + (j >> 5)] = bits;
            bits = 0;
          }
        }
        if (MODE == kSkip && gt == 0) {
          st_release_shared(smem_u32(&ctl.dec[x][j % kDecRing]), ((j + 1) << 1) | (skip ? 1 : 0));
        }
      }
      if (skip) {  // nothing to hand over: P-ready counts kept tiles only
        ++nskip;
        continue;
      }

      // Kept tile: online softmax update. Every earlier MMA into O_X has
      // completed (S_X(j) completing implies it), so O_X may be rescaled here.
      const float m_new = fmaxf(m_true, tmax);
      m_true = m_new;
      float alpha = 1.f;
      // Reference of the exponentials. bf16 P: m_used, moved to m_true only
      // once m_true passes it by kRescaleThreshold, so O is rescaled rarely.
      // E4M3 P: an integer r >= m_true (held in m_used), raised to
      // ceil(m_true) as soon as m_true passes it, so that P = 2^(s2 - r + 8)
      // lies in (0, 256], inside E4M3's range, and every rescale factor
      // 2^(r_old - r_new) is an exact power of two.
      const bool up = F8V ? m_new > m_used : m_new > m_used + kRescaleThreshold;
      if (__any_sync(kFull, up)) {
        if (F8V) {
          if (up) {
            const float r_new = ceilf(m_new);
            const float e = m_used - r_new;  // a negative integer, or -inf before the first kept tile
            alpha = e < -126.f ? 0.f : __int_as_float((static_cast<int>(e) + 127) << 23);
            m_used = r_new;
          }
        } else {
          alpha = ex2_approx(m_used - m_new);  // 0 before the first kept tile
          m_used = m_new;
        }
        if (kept > 0) {
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t o[32];
            tmem_ld_x32(lane_base + col_o + ch * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st_x32(lane_base + col_o + ch * 32, o);
          }
        }
      }
      l *= alpha;
      const float bias = F8V ? 8.f - m_used : -m_used;
      const float2 c2 = make_float2(c, c), nm2 = make_float2(bias, bias);
      float2 rs[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      uint32_t lo[64];
      tmem_ld_x64_async(lane_base + col_s, lo);  // lands while the upper half is exponentiated
      if (F8V) {
        // E4M3 P, four consecutive kv per column: kv [64,128) stored to
        // columns [64,80) as soon as computed (those S columns have been
        // read), kv [0,64) to columns [0,16) once the lower half is back.
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 a0 = ffma2(make_float2(__uint_as_float(hi[4 * i]), __uint_as_float(hi[4 * i + 1])), c2, nm2);
          const float2 a1 =
              ffma2(make_float2(__uint_as_float(hi[4 * i + 2]), __uint_as_float(hi[4 * i + 3])), c2, nm2);
          const float2 e0 = make_float2(ex2_approx(a0.x), ex2_approx(a0.y));
          const float2 e1 = make_float2(ex2_approx(a1.x), ex2_approx(a1.y));
          rs[0] = fadd2(rs[0], e0);
          rs[1] = fadd2(rs[1], e1);
          pk[i] = pack_e4m3x2(e0.x, e0.y) | (pack_e4m3x2(e1.x, e1.y) << 16);
        }
        tmem_st_x16(lane_base + col_s + 64, pk);
        warp_arrive(p_hi(x), lane);
        tmem_wait_ld_tied(lo);
        if (valid < 64) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (i >= valid) lo[i] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 a0 = ffma2(make_float2(__uint_as_float(lo[4 * i]), __uint_as_float(lo[4 * i + 1])), c2, nm2);
          const float2 a1 =
              ffma2(make_float2(__uint_as_float(lo[4 * i + 2]), __uint_as_float(lo[4 * i + 3])), c2, nm2);
          const float2 e0 = make_float2(ex2_approx(a0.x), ex2_approx(a0.y));
          const float2 e1 = make_float2(ex2_approx(a1.x), ex2_approx(a1.y));
          rs[0] = fadd2(rs[0], e0);
          rs[1] = fadd2(rs[1], e1);
          pk[i] = pack_e4m3x2(e0.x, e0.y) | (pack_e4m3x2(e1.x, e1.y) << 16);
        }
        tmem_st_x16(lane_base + col_s, pk);
      } else {
        // Packed P: bf16 pairs of consecutive kv columns; the upper half's
        // pairs go to columns [64,96) right away (the issuer starts on them),
        // the lower half's to [0,32) once they are computed.
        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 a = ffma2(make_float2(__uint_as_float(hi[2 * i]), __uint_as_float(hi[2 * i + 1])), c2, nm2);
          const float2 e = make_float2(ex2_approx(a.x), ex2_approx(a.y));
          rs[i & 1] = fadd2(rs[i & 1], e);
          pk[32 + i] = pack_bf16x2(e.x, e.y);
        }
        tmem_st_x32(lane_base + col_s + 64, reinterpret_cast<const uint32_t(&)[32]>(pk[32]));
        warp_arrive(p_hi(x), lane);
        tmem_wait_ld_tied(lo);
        if (valid < 64) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (i >= valid) lo[i] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 a = ffma2(make_float2(__uint_as_float(lo[2 * i]), __uint_as_float(lo[2 * i + 1])), c2, nm2);
          const float2 e = make_float2(ex2_approx(a.x), ex2_approx(a.y));
          rs[i & 1] = fadd2(rs[i & 1], e);
          pk[i] = pack_bf16x2(e.x, e.y);
        }
        // Both halves of S_X are in registers by now: P_X may overwrite them.
        tmem_st_x32(lane_base + col_s, reinterpret_cast<const uint32_t(&)[32]>(pk[0]));
      }
      l += (rs[0].x + rs[1].x) + (rs[0].y + rs[1].y);
      warp_arrive(p_ready(x), lane);
      ++kept;
    }

    // A warp that left the loop on an error arrives once on its group's vote
    // barrier, so the group's other warps cannot be left waiting at it: the
    // barrier is a full barrier per tile, so no warp is more than one instance away.
    if (!ok && (MODE != kDense || EX)) named_barrier_arrive(vote_bar, 128);

    // Epilogue: O_X / l -> bf16, masked row stores; per-unit counters.
    if (ok) ok = warp_wait(o_final, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const float inv_l = F8V ? p.v_scale / l : 1.0f / l;
      __nv_bfloat16* orow =
          p.out + (static_cast<int64_t>(seq_start + qb * kBM + row) * p.num_heads + head) * static_cast<int64_t>(D);
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld_x32(lane_base + col_o + ch * 32, o);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (MODE == kCalib) {  // add over the 16 lanes that share thresholds; lanes 0 and 16 store
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          int v = cal_cnt[m];
#pragma unroll
          for (int o = 1; o < 16; o <<= 1) v += __shfl_xor_sync(kFull, v, o);
          const int k = (gt >> 4) + 8 * m;
          if ((lane & 15) == 0 && k < p.n_cal) p.counts[unit * p.n_cal + k] = v;
        }
      }
      if (gt == 0 && p.skip_counter) p.skip_counter[unit] = nskip;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Runs the kernels' bounded mbarrier wait on a barrier that nothing arrives
// on, with a short limit: the wait must give up, raise the abort flag and
// record the timeout in the status word, and the kernel must return.
__global__ void wait_timeout_check_kernel(uint64_t limit_ns, int* result) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(smem_u32(&bar), 1);
  fence_mbar_init();
  const uint64_t t0 = globaltimer_ns();
  const bool completed = wait_bar(smem_u32(&bar), 0, &abort_flag, limit_ns);
  result[0] = completed ? 1 : 0;
  result[1] = abort_flag;
  result[2] = static_cast<int>((globaltimer_ns() - t0) / 1000);  // microseconds waited
}

// Clears the given bits of the status word atomically (ssa_get_error).
__global__ void status_clear_kernel(int bits) { atomicAnd(&g_status, ~bits); }

// ----------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// [total_tokens, H, D] viewed as a 3-D tensor (d, head, token) of bf16 (or
// of bytes, for E4M3); box of 128 bytes of d x 1 head x 128 tokens with
// 128-byte swizzle. Rows past total_tokens read as zero.
bool make_tensor_map(CUtensorMap* map, const void* base, int total_tokens, int H, int D, bool bytes) {
  auto encode = encode_fn();
  if (!encode) return false;
  const cuuint64_t esize = bytes ? 1 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(total_tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * esize, static_cast<cuuint64_t>(H) * D * esize};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esize), 1, static_cast<cuuint32_t>(kBN)};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(map, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Call {
  const void *q, *k, *v;
  const int32_t* cu;
  int batch, total_tokens, max_seqlen, H, D;
  float softmax_scale;
  void* out;
  cudaStream_t stream;
  bool f8 = false;              // Q and K are E4M3 bytes
  bool f8v = false;             // V is E4M3 bytes too (and P is rounded to E4M3)
  double qk_descale = 1.0;      // q_descale * k_descale (E4M3 only)
  float v_descale = 1.0f;       // multiplies the output when V is E4M3
};

// True when `p` is device (or managed) memory of the current device: a host
// pointer handed to a kernel or a tensor map would fault the GPU, so every
// pointer the kernels touch is checked before a launch.
bool on_current_device(const void* ptr) {
  if (!ptr) return false;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaPointerAttributes attr{};
  if (cudaPointerGetAttributes(&attr, ptr) != cudaSuccess) {
    cudaGetLastError();  // clear the error this query may leave behind
    return false;
  }
  return (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged) && attr.device == dev;
}

// Every non-null pointer of `ptrs` lives on the current device.
int check_device_pointers(std::initializer_list<const void*> ptrs) {
  for (const void* ptr : ptrs)
    if (ptr && !on_current_device(ptr)) return SSA_ERR_INVALID_ARG;
  return SSA_OK;
}

// Host-side argument check. total_tokens == 0 is a valid no-op whatever the
// data pointers are (an empty batch has no storage).
int validate(const Call& a) {
  if (!a.cu || a.batch < 1 || a.total_tokens < 0 || a.max_seqlen < 0 || a.H < 1 || a.H > 65535)
    return SSA_ERR_INVALID_ARG;
  if (std::isnan(a.softmax_scale) || std::isinf(a.softmax_scale)) return SSA_ERR_INVALID_ARG;
  if (a.D != 64 && a.D != 128) return SSA_ERR_UNSUPPORTED;
  if (a.f8 && a.D != 128) return SSA_ERR_UNSUPPORTED;  // E4M3 rows of 128 B: one swizzle atom per row
  if (a.f8 && !(a.qk_descale > 0.0 && std::isfinite(a.qk_descale))) return SSA_ERR_INVALID_ARG;
  if (a.f8v && !(a.v_descale > 0.f && std::isfinite(a.v_descale))) return SSA_ERR_INVALID_ARG;
  if (a.total_tokens == 0) return SSA_OK;
  if (!a.q || !a.k || !a.v || !a.out) return SSA_ERR_INVALID_ARG;
  for (const void* ptr : {a.q, a.k, a.v, static_cast<const void*>(a.out)})
    if (reinterpret_cast<uintptr_t>(ptr) & 15u) return SSA_ERR_UNSUPPORTED;
  return check_device_pointers({a.q, a.k, a.v, a.out, a.cu});
}

Params base_params(const Call& a) {
  Params p{};
  p.cu_seqlens = a.cu;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.batch = a.batch;
  p.total_tokens = a.total_tokens;
  p.num_heads = a.H;
  p.max_tiles = (a.max_seqlen + kBN - 1) / kBN;
  p.bitmap_words = (p.max_tiles + 31) / 32;
  p.nq_check = -1;
  double scale = a.softmax_scale > 0.f ? static_cast<double>(a.softmax_scale) : 1.0 / std::sqrt(static_cast<double>(a.D));
  if (a.f8) scale = scale * a.qk_descale;  // E4M3 codes carry the per-tensor scales of Q and K
  p.c = static_cast<float>(scale * 1.4426950408889634073599246810019);
  p.v_scale = a.f8v ? a.v_descale : 1.0f;
  return p;
}

template <int D, int MODE, bool EX, int PREC>
int launch(const Call& a, const Params& p) {
  CUtensorMap tq, tk, tv;
  if (!make_tensor_map(&tq, a.q, a.total_tokens, a.H, D, PREC >= kQK8) ||
      !make_tensor_map(&tk, a.k, a.total_tokens, a.H, D, PREC >= kQK8) ||
      !make_tensor_map(&tv, a.v, a.total_tokens, a.H, D, PREC == kQKV8)) {
    t_last_cuda_error = "cuTensorMapEncodeTiled failed or the driver entry point is unavailable";
    return SSA_ERR_CUDA;
  }
  auto kernel = ssa_attention_kernel<D, MODE, EX, PREC>;
  constexpr int smem = Layout<D, PREC>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e);
  // one CTA per pair of query blocks: sum over sequences of ceil(S_b / 256) <= ceil(T / 256) + batch
  const dim3 grid(static_cast<unsigned>((a.total_tokens + 2 * kBM - 1) / (2 * kBM) + a.batch),
                  static_cast<unsigned>(a.H));
  kernel<<<grid, kThreads, smem, a.stream>>>(tq, tk, tv, p);
  e = cudaGetLastError();
  return e == cudaSuccess ? SSA_OK : cuda_fail(e);
}

template <int MODE, bool EX>
int dispatch_d(const Call& a, const Params& p) {
  if (a.f8v) return launch<128, MODE, EX, kQKV8>(a, p);
  if (a.f8) return launch<128, MODE, EX, kQK8>(a, p);
  return a.D == 64 ? launch<64, MODE, EX, kBf16>(a, p) : launch<128, MODE, EX, kBf16>(a, p);
}

// y = E4M3(fp32(x * inv_scale)), round to nearest even, saturating to +-448;
// eight elements per thread (16-byte loads, 8-byte stores), a scalar tail.
__global__ void quantize_e4m3_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ y, int64_t n,
                                     float inv_scale) {
  auto cvt2 = [](float lo, float hi) -> uint32_t {
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
  };
  const int64_t groups = n / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < groups; g += stride) {
    const uint4 v = reinterpret_cast<const uint4*>(x)[g];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __uint_as_float(w[i] << 16) * inv_scale;
      const float hi = __uint_as_float(w[i] & 0xFFFF0000u) * inv_scale;
      o[i >> 1] |= cvt2(lo, hi) << ((i & 1) * 16);
    }
    reinterpret_cast<uint2*>(y)[g] = make_uint2(o[0], o[1]);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (int64_t i = groups * 8; i < n; ++i) {
      const float f = __bfloat162float(x[i]) * inv_scale;
      y[i] = static_cast<uint8_t>(cvt2(f, 0.f) & 0xFFu);
    }
  }
}

int fwd_impl(const Call& a, float tsf, int32_t* skip_counter, int num_qblocks, uint32_t* bitmap, float* tile_stat) {
  int rc = validate(a);
  if (rc != SSA_OK) return rc;
  if (std::isnan(tsf) || std::isinf(tsf)) return SSA_ERR_INVALID_ARG;
  if ((bitmap || tile_stat) && a.max_seqlen < 1) return SSA_ERR_INVALID_ARG;
  const bool per_unit = skip_counter || bitmap || tile_stat;
  if (per_unit && num_qblocks < 0) return SSA_ERR_INVALID_ARG;
  if (a.total_tokens == 0) return SSA_OK;
  if ((rc = check_device_pointers({skip_counter, bitmap, tile_stat})) != SSA_OK) return rc;
  Params p = base_params(a);
  p.nq_check = per_unit ? num_qblocks : -1;
  p.skip_counter = skip_counter;
  p.bitmap = bitmap;
  p.tile_stat = tile_stat;
  p.tsf = tsf;
  const bool ex = bitmap || tile_stat;
  if (tsf > 0.f) return ex ? dispatch_d<kSkip, true>(a, p) : dispatch_d<kSkip, false>(a, p);
  return ex ? dispatch_d<kDense, true>(a, p) : dispatch_d<kDense, false>(a, p);
}

}  // namespace
}  // namespace ssa

using namespace ssa;

extern "C" int ssa_fwd_fp8(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                           int total_tokens, int max_seqlen, int num_heads, int head_dim, float softmax_scale,
                           float q_descale, float k_descale, float threshold_scale_factor, void* out,
                           int32_t* skip_counter, int num_qblocks, uint32_t* decision_bitmap, float* tile_stat,
                           void* stream) {
  Call a{q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, num_heads, head_dim, softmax_scale, out,
         static_cast<cudaStream_t>(stream)};
  if (!(q_descale > 0.f) || !(k_descale > 0.f) || std::isinf(q_descale) || std::isinf(k_descale))
    return SSA_ERR_INVALID_ARG;
  a.f8 = true;
  a.qk_descale = static_cast<double>(q_descale) * static_cast<double>(k_descale);
  return fwd_impl(a, threshold_scale_factor, skip_counter, num_qblocks, decision_bitmap, tile_stat);
}

extern "C" int ssa_fwd_fp8_qkv(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                               int total_tokens, int max_seqlen, int num_heads, int head_dim, float softmax_scale,
                               float q_descale, float k_descale, float v_descale, float threshold_scale_factor,
                               void* out, int32_t* skip_counter, int num_qblocks, uint32_t* decision_bitmap,
                               float* tile_stat, void* stream) {
  Call a{q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, num_heads, head_dim, softmax_scale, out,
         static_cast<cudaStream_t>(stream)};
  if (!(q_descale > 0.f) || !(k_descale > 0.f) || std::isinf(q_descale) || std::isinf(k_descale))
    return SSA_ERR_INVALID_ARG;
  a.f8 = a.f8v = true;
  a.qk_descale = static_cast<double>(q_descale) * static_cast<double>(k_descale);
  a.v_descale = v_descale;
  return fwd_impl(a, threshold_scale_factor, skip_counter, num_qblocks, decision_bitmap, tile_stat);
}

extern "C" int ssa_quantize_fp8(const void* x, void* y, int64_t n, float inv_scale, void* stream) {
  if (n < 0 || !(inv_scale > 0.f) || std::isinf(inv_scale)) return SSA_ERR_INVALID_ARG;
  if (n == 0) return SSA_OK;
  if (!x || !y) return SSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(y) & 7u)) return SSA_ERR_UNSUPPORTED;
  if (const int rc = check_device_pointers({x, y}); rc != SSA_OK) return rc;
  const int64_t groups = n / 8;
  const int threads = 256;
  const int64_t want = (groups + threads - 1) / threads;
  const unsigned blocks = static_cast<unsigned>(want < 1 ? 1 : (want > 148 * 16 ? 148 * 16 : want));
  quantize_e4m3_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<uint8_t*>(y), n, inv_scale);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SSA_OK : cuda_fail(e);
}

extern "C" int ssa_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                       int total_tokens, int max_seqlen, int num_heads, int head_dim, float softmax_scale,
                       float threshold_scale_factor, void* out, int32_t* skip_counter, int num_qblocks,
                       void* stream) {
  const Call a{q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, num_heads, head_dim, softmax_scale, out,
               static_cast<cudaStream_t>(stream)};
  return fwd_impl(a, threshold_scale_factor, skip_counter, num_qblocks, nullptr, nullptr);
}

extern "C" int ssa_fwd_ex(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                          int total_tokens, int max_seqlen, int num_heads, int head_dim, float softmax_scale,
                          float threshold_scale_factor, void* out, int32_t* skip_counter, int num_qblocks,
                          uint32_t* decision_bitmap, float* tile_stat, void* stream) {
  const Call a{q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, num_heads, head_dim, softmax_scale, out,
               static_cast<cudaStream_t>(stream)};
  return fwd_impl(a, threshold_scale_factor, skip_counter, num_qblocks, decision_bitmap, tile_stat);
}

namespace ssa {
namespace {
int calibrate_impl(const Call& a, const float* thresholds, int n_thresholds, int32_t* counts, int num_qblocks,
                   float* tile_stat) {
  int rc = validate(a);
  if (rc != SSA_OK) return rc;
  if (!thresholds || !counts || n_thresholds < 1 || n_thresholds > SSA_MAX_THRESHOLDS || num_qblocks < 0)
    return SSA_ERR_INVALID_ARG;
  for (int i = 0; i < n_thresholds; ++i)
    if (!(thresholds[i] > 0.f) || std::isinf(thresholds[i])) return SSA_ERR_INVALID_ARG;
  if (tile_stat && a.max_seqlen < 1) return SSA_ERR_INVALID_ARG;
  if (a.total_tokens == 0) return SSA_OK;
  if ((rc = check_device_pointers({counts, tile_stat})) != SSA_OK) return rc;
  Params p = base_params(a);
  p.nq_check = num_qblocks;
  p.counts = counts;
  p.tile_stat = tile_stat;
  p.n_cal = n_thresholds;
  for (int i = 0; i < n_thresholds; ++i) p.Lcal[i] = static_cast<float>(std::log2(static_cast<double>(thresholds[i])));
  return tile_stat ? dispatch_d<kCalib, true>(a, p) : dispatch_d<kCalib, false>(a, p);
}
}  // namespace
}  // namespace ssa

extern "C" int ssa_calibrate(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                             int total_tokens, int max_seqlen, int num_heads, int head_dim, float softmax_scale,
                             const float* thresholds, int n_thresholds, void* out, int32_t* counts, int num_qblocks,
                             void* stream) {
  const Call a{q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, num_heads, head_dim, softmax_scale, out,
               static_cast<cudaStream_t>(stream)};
  return calibrate_impl(a, thresholds, n_thresholds, counts, num_qblocks, nullptr);
}

extern "C" int ssa_calibrate_ex(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                                int total_tokens, int max_seqlen, int num_heads, int head_dim, float softmax_scale,
                                const float* thresholds, int n_thresholds, void* out, int32_t* counts,
                                int num_qblocks, float* tile_stat, void* stream) {
  const Call a{q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, num_heads, head_dim, softmax_scale, out,
               static_cast<cudaStream_t>(stream)};
  return calibrate_impl(a, thresholds, n_thresholds, counts, num_qblocks, tile_stat);
}

extern "C" int ssa_calibrate_fp8(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int batch,
                                 int total_tokens, int max_seqlen, int num_heads, int head_dim, float softmax_scale,
                                 float q_descale, float k_descale, const float* thresholds, int n_thresholds,
                                 void* out, int32_t* counts, int num_qblocks, void* stream) {
  Call a{q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, num_heads, head_dim, softmax_scale, out,
         static_cast<cudaStream_t>(stream)};
  if (!(q_descale > 0.f) || !(k_descale > 0.f) || std::isinf(q_descale) || std::isinf(k_descale))
    return SSA_ERR_INVALID_ARG;
  a.f8 = true;
  a.qk_descale = static_cast<double>(q_descale) * static_cast<double>(k_descale);
  return calibrate_impl(a, thresholds, n_thresholds, counts, num_qblocks, nullptr);
}

extern "C" int ssa_calibrate_fp8_qkv(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                                     int batch, int total_tokens, int max_seqlen, int num_heads, int head_dim,
                                     float softmax_scale, float q_descale, float k_descale, float v_descale,
                                     const float* thresholds, int n_thresholds, void* out, int32_t* counts,
                                     int num_qblocks, void* stream) {
  Call a{q, k, v, cu_seqlens, batch, total_tokens, max_seqlen, num_heads, head_dim, softmax_scale, out,
         static_cast<cudaStream_t>(stream)};
  if (!(q_descale > 0.f) || !(k_descale > 0.f) || std::isinf(q_descale) || std::isinf(k_descale))
    return SSA_ERR_INVALID_ARG;
  a.f8 = a.f8v = true;
  a.qk_descale = static_cast<double>(q_descale) * static_cast<double>(k_descale);
  a.v_descale = v_descale;
  return calibrate_impl(a, thresholds, n_thresholds, counts, num_qblocks, nullptr);
}

extern "C" const char* ssa_last_cuda_error(void) { return t_last_cuda_error; }

extern "C" int ssa_wait_timeout_check(int* result, int64_t limit_ns, void* stream) {
  if (!result || limit_ns <= 0 || limit_ns > 1000000000) return SSA_ERR_INVALID_ARG;
  if (const int rc = check_device_pointers({result}); rc != SSA_OK) return rc;
  wait_timeout_check_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(limit_ns), result);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SSA_OK : cuda_fail(e);
}

extern "C" int ssa_get_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  if (v != 0) {  // clear exactly the bits read: a bit another stream sets meanwhile stays for the next call
    status_clear_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(v);
    if ((e = cudaGetLastError()) != cudaSuccess || (e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream))) !=
                                                       cudaSuccess)
      return cuda_fail(e);
  }
  if (v & kStatusTimeout) return SSA_ERR_TIMEOUT;
  if (v & kStatusDeviceArg) return SSA_ERR_DEVICE_ARG;
  return SSA_OK;
}
