// moe_kernels.cu -- routing, capacity-limited slot assignment and the HBM-bound data movement
// of the MoE block (sm_100a).
//
//   route_topk      one warp per token: top-k of float32 logits + bias (ties to the lower
//                   expert index), softmax gates of the chosen unbiased logits, load histogram
//                   ("Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播", §2.2)
//   slot scan       deterministic two-level prefix scan in (token, rank) order: sender slot
//                   per (destination, wave) pool capped at C_s, receiver slot per expert among
//                   sender-kept rows capped at C_r ("Marin начинает открытое обучение
//                   MoE-модели с 535 млрд параметров", §2: caps 1.10 / 1.15, drops counted
//                   separately)
//   pack            sender: z rows into the fixed pools with the expert id in a 16-byte row
//                   header (same page, §2: one pool per receiving GPU, ids in the payload)
//   unpack          receiver: reads only the pools; ranks rows of each local expert by the
//                   packed id, keeps the first C_r, gathers them per expert
//   combine         r_t = sum_j kept g_tj Y[e_tj][rslot_tj], fixed j order, fp32 accumulation
//   combine_bwd     dY = g dr on kept rows, dg = <dr, Y>
//   undispatch      dz_routed = sum_j kept dX, and the softmax backward to the logits
//   bias_update     zero-mean sign step from the histogram
// All data movement uses 16-byte vector loads and stores on row-contiguous data.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

#define MOE_TRY_K(x)               \
  do {                             \
    moe_status_t _s = (x);         \
    if (_s != MOE_OK) return _s;   \
  } while (0)

namespace {

constexpr int kMaxE = 1024;

__device__ __forceinline__ bool better(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

// ---------------------------------------------------------------------- routing

// Sort 32 distinct (score, expert, raw) keys across the warp, best first under `better`
// (bitonic network over the lanes: lane 0 ends with the best).
__device__ __forceinline__ void warp_sort_best_first(float& v, int& e, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const float pv = __shfl_xor_sync(0xffffffffu, v, stride);
      const int pe = __shfl_xor_sync(0xffffffffu, e, stride);
      const bool lower = (lane & stride) == 0;
      const bool best_first = (lane & size) == 0;  // direction of this block of the network
      const bool pb = better(pv, pe, v, e);
      if ((lower == best_first) ? pb : !pb) {
        v = pv;
        e = pe;
      }
    }
  }
}

// the same network carrying a third value (the raw logit) with each key
__device__ __forceinline__ void warp_sort_best_first(float& v, int& e, float& r, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const float pv = __shfl_xor_sync(0xffffffffu, v, stride);
      const int pe = __shfl_xor_sync(0xffffffffu, e, stride);
      const float pr = __shfl_xor_sync(0xffffffffu, r, stride);
      const bool lower = (lane & stride) == 0;
      const bool best_first = (lane & size) == 0;  // direction of this block of the network
      const bool pb = better(pv, pe, v, e);
      if ((lower == best_first) ? pb : !pb) {
        v = pv;
        e = pe;
        r = pr;
      }
    }
  }
}

// One warp per token.  The k-th best of the 32 lane maxima bounds the k-th best score from
// below (the k best lane maxima are k distinct scores at or above it), so the top k are
// among the scores not worse than it; those candidates (usually a few more than k) are
// gathered with ballots and sorted across the warp.  More than 32 candidates (many equal
// scores) take k rounds of warp arg-max instead.  Either way the result is the exact top k
// under (score descending, expert ascending), in that order.
template <int VPL>
__global__ void __launch_bounds__(256, 3) route_topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E,
                                  int k, int32_t* __restrict__ idx_out, float* __restrict__ gate_out,
                                  int32_t* __restrict__ hist, int32_t* __restrict__ nan_count) {
  // hist == nullptr: the histogram is left to the slot scan, which counts every assignment
  __shared__ int sh_hist[kMaxE];
  __shared__ float sh_cv[8][32], sh_cr[8][32];  // candidates of each warp (blocks of <= 8 warps)
  __shared__ int sh_ce[8][32];
  if (hist != nullptr)
    for (int e = threadIdx.x; e < E; e += blockDim.x) sh_hist[e] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int warps = blockDim.x >> 5;
  const int gw = blockIdx.x * warps + wib;
  const int nw = gridDim.x * warps;
  const unsigned lt_mask = (1u << lane) - 1u;
  float bsv[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = i * 32 + lane;
    bsv[i] = e < E ? bias[e] : 0.0f;
  }
  int nan_local = 0;
  // each warp walks tokens gw, gw + nw, ...; the next token's logits load while this
  // token's experts are selected
  float nxt[VPL];
  auto load_row = [&](int t) {
    const float* row = logits + static_cast<long long>(t) * E;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = i * 32 + lane;
      nxt[i] = e < E ? __ldcs(row + e) : 0.0f;
    }
  };
  if (gw < T) load_row(gw);
  for (int t = gw; t < T; t += nw) {
    float raw[VPL], sc[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) raw[i] = nxt[i];
    if (t + nw < T) load_row(t + nw);
    float mv = -INFINITY;
    int me = 0x7fffffe0 + lane;  // a lane with no expert ranks below every expert
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = i * 32 + lane;
      sc[i] = __fadd_rn(raw[i], bsv[i]);
      if (e < E && isnan(sc[i])) {
        ++nan_local;          // input error, counted; the expert ranks last
        sc[i] = -INFINITY;
      }
      if (e < E && better(sc[i], e, mv, me)) {
        mv = sc[i];
        me = e;
      }
    }
    // threshold: the k-th best lane maximum
    float tv = mv;
    int te = me;
    warp_sort_best_first(tv, te, lane);
    tv = __shfl_sync(0xffffffffu, tv, k - 1);
    te = __shfl_sync(0xffffffffu, te, k - 1);
    // candidates: scores not worse than the threshold
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = i * 32 + lane;
      cnt += (e < E && !better(tv, te, sc[i], e)) ? 1 : 0;
    }
    int total = cnt;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) total += __shfl_xor_sync(0xffffffffu, total, off);
    float my_raw = 0.0f;  // lane j < k keeps the raw logit of its rank-j choice
    int my_e = 0;
    if (total <= 32) {
      int base = 0;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int e = i * 32 + lane;
        const bool c = e < E && !better(tv, te, sc[i], e);
        const unsigned m = __ballot_sync(0xffffffffu, c);
        if (c) {
          const int pos = base + __popc(m & lt_mask);
          sh_cv[wib][pos] = sc[i];
          sh_ce[wib][pos] = e;
          sh_cr[wib][pos] = raw[i];
        }
        base += __popc(m);
      }
      __syncwarp();
      float cv = -INFINITY, cr = 0.0f;
      int ce = 0x7fffffe0 + lane;
      if (lane < total) {
        cv = sh_cv[wib][lane];
        ce = sh_ce[wib][lane];
        cr = sh_cr[wib][lane];
      }
      __syncwarp();
      warp_sort_best_first(cv, ce, cr, lane);
      my_raw = cr;
      my_e = ce;
    } else {
      unsigned chosen = 0;
      for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
          const int e = i * 32 + lane;
          if (e < E && !((chosen >> i) & 1u) && better(sc[i], e, bv, be)) {
            bv = sc[i];
            be = e;
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
          const int oe = __shfl_xor_sync(0xffffffffu, be, off);
          if (better(ov, oe, bv, be)) {
            bv = ov;
            be = oe;
          }
        }
        // be is now the same on every lane; its owner marks it and shares the raw logit
        const int owner = be & 31;
        const int slot = be >> 5;
        float r = 0.0f;
#pragma unroll
        for (int i = 0; i < VPL; ++i)
          if (i == slot && lane == owner) {
            chosen |= 1u << i;
            r = raw[i];
          }
        r = __shfl_sync(0xffffffffu, r, owner);
        if (lane == j) {
          my_raw = r;
          my_e = be;
        }
      }
    }
    // softmax over the k chosen raw logits (lanes 0..k-1)
    float m = lane < k ? my_raw : -INFINITY;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float ex = lane < k ? expf(my_raw - m) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < k) {
      idx_out[static_cast<long long>(t) * k + lane] = my_e;
      gate_out[static_cast<long long>(t) * k + lane] = ex / sum;
      if (hist != nullptr && my_e >= 0 && my_e < E) atomicAdd(&sh_hist[my_e], 1);
    }
  }
  if (nan_local && nan_count != nullptr) atomicAdd(nan_count, nan_local);
  __syncthreads();
  if (hist != nullptr)
    for (int e = threadIdx.x; e < E; e += blockDim.x)
      if (sh_hist[e]) atomicAdd(&hist[e], sh_hist[e]);
}

// ---------------------------------------------------------------------- slot scan
//
// Chunks of kScanTokensPerChunk tokens (their k assignments, in (t, j) order).
//   A  count per chunk and pool                      cnt_pool[p][c]
//   B  exclusive scan over chunks per pool            base_pool[p][c]
//   C  sender slot = base + rank in chunk (warp-ordered); count sender-kept per expert
//   D  exclusive scan over chunks per expert          base_exp[e][c]
//   E  receiver slot = base + rank among kept in chunk; counters
// Each per-chunk pass is one warp walking its chunk 32 assignments at a time, so the
// ranks follow the visiting order exactly.

__device__ __forceinline__ int pool_of(int e, int L, int P, int W) { return (e / L) * W + (e % L) / P; }

__global__ void scan_count_pools(const int32_t* __restrict__ idx, int A_total, int chunk_assign, int n_chunks,
                                 int L, int P, int W, int NP, int E, int32_t* __restrict__ cnt_pool) {
  extern __shared__ int sh[];
  const int c = blockIdx.x;
  for (int p = threadIdx.x; p < NP; p += blockDim.x) sh[p] = 0;
  __syncthreads();
  const int a0 = c * chunk_assign;
  const int a1 = min(A_total, a0 + chunk_assign);
  for (int a = a0 + threadIdx.x; a < a1; a += blockDim.x) {
    const int e = idx[a];
    if (e >= 0 && e < E) atomicAdd(&sh[pool_of(e, L, P, W)], 1);
  }
  __syncthreads();
  for (int p = threadIdx.x; p < NP; p += blockDim.x) cnt_pool[static_cast<long long>(p) * n_chunks + c] = sh[p];
}

// exclusive scan of each row of a [rows][n] int array, one block per row, restarted every
// seg elements (seg divides n; seg = n: one segment).  Segment s of row r: its total goes
// to totals[s * rows + r] (optional), clamped at cap into clamp_out[s * rows + r] (optional).
__global__ void scan_rows(int32_t* __restrict__ data, int n, int32_t* __restrict__ totals, int cap,
                          int32_t* __restrict__ clamp_out, int seg) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  int32_t* row = data + static_cast<long long>(blockIdx.x) * n;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  for (int s0 = 0; s0 < n; s0 += seg) {
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int s1 = min(n, s0 + seg);
    for (int base = s0; base < s1; base += blockDim.x) {
      const int i = base + threadIdx.x;
      const int v = i < s1 ? row[i] : 0;
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (lane == 31) warp_tot[warp] = incl;
      __syncthreads();
      int before = carry;
      for (int w = 0; w < warp; ++w) before += warp_tot[w];
      if (i < s1) row[i] = before + incl - v;
      __syncthreads();
      if (threadIdx.x == blockDim.x - 1) carry = before + incl;
      __syncthreads();
      (void)nwarp;
    }
    if (threadIdx.x == 0) {
      const long long o = static_cast<long long>(s0 / seg) * gridDim.x + blockIdx.x;
      if (totals) totals[o] = carry;
      if (clamp_out) clamp_out[o] = carry < cap ? carry : cap;
    }
    __syncthreads();
  }
}

// pass C: one warp per chunk
// rows of 32 assignments whose loads a scan warp issues before ranking them
constexpr int kScanBatch = 8;

__global__ void scan_sender_slots(const int32_t* __restrict__ idx, int A_total, int chunk_assign, int n_chunks,
                                  int L, int P, int W, int NP, int E, int Cs,
                                  const int32_t* __restrict__ base_pool, int32_t* __restrict__ slot,
                                  int32_t* __restrict__ cnt_exp, int32_t* __restrict__ status) {
  extern __shared__ int sh[];  // per warp: NP running counters + E kept counters
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int c = blockIdx.x * (blockDim.x >> 5) + wib;
  int* run = sh + wib * (NP + E);
  int* kept = run + NP;
  for (int i = lane; i < NP + E; i += 32) run[i] = 0;
  __syncwarp();
  if (c >= n_chunks) return;
  const int a0 = c * chunk_assign;
  const int a1 = min(A_total, a0 + chunk_assign);
  // up to kScanBatch rows of 32 assignments at a time: their expert ids, then their pools'
  // bases, are loaded before the rows are ranked in order
  for (int it0 = a0; it0 < a1; it0 += 32 * kScanBatch) {
    int eb[kScanBatch], bb[kScanBatch];
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u) {
      const int a = it0 + 32 * u + lane;
      eb[u] = a < a1 ? idx[a] : 0;
    }
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u) {
      const int a = it0 + 32 * u + lane;
      const bool ok = a < a1 && eb[u] >= 0 && eb[u] < E;
      bb[u] = ok ? base_pool[static_cast<long long>(pool_of(eb[u], L, P, W)) * n_chunks + c] : 0;
    }
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u) {
      if (it0 + 32 * u >= a1) break;  // warp-uniform
      const int a = it0 + 32 * u + lane;
      const int e_raw = eb[u];
      const bool bad = a < a1 && (e_raw < 0 || e_raw >= E);
      if (bad) {
        atomicCAS(status, 0, MOE_ERR_INVALID_ARG);
        slot[2LL * a] = -1;
      }
      const bool valid = a < a1 && !bad;
      const int e = valid ? e_raw : 0;
      const int p = valid ? pool_of(e, L, P, W) : -1 - lane;
      const unsigned act = __ballot_sync(0xffffffffu, valid);
      const unsigned peers = __match_any_sync(0xffffffffu, p) & act;
      const int rank = __popc(peers & ((1u << lane) - 1u));
      int s = -1;
      if (valid) {
        s = bb[u] + run[p] + rank;
      }
      __syncwarp();
      if (valid && rank == __popc(peers) - 1) run[p] += __popc(peers);  // last of its group
      if (valid) {
        const bool sk = s < Cs;
        slot[2LL * a] = sk ? s : -1;
        if (sk) atomicAdd(&kept[e], 1);
      }
      __syncwarp();
    }
  }
  __syncwarp();
  for (int e = lane; e < E; e += 32) cnt_exp[static_cast<long long>(e) * n_chunks + c] = kept[e];
}

// pass E: one warp per chunk
__global__ void scan_receiver_slots(const int32_t* __restrict__ idx, int A_total, int chunk_assign, int n_chunks,
                                    int E, int Cr, const int32_t* __restrict__ base_exp,
                                    int32_t* __restrict__ slot, int32_t* __restrict__ stats_kept_e,
                                    int32_t* __restrict__ stats_ds_e, int32_t* __restrict__ stats_dr_e) {
  extern __shared__ int sh[];  // per warp: E running counters
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int c = blockIdx.x * (blockDim.x >> 5) + wib;
  int* run = sh + wib * E;
  for (int i = lane; i < E; i += 32) run[i] = 0;
  __syncwarp();
  if (c >= n_chunks) return;
  const int a0 = c * chunk_assign;
  const int a1 = min(A_total, a0 + chunk_assign);
  // as in the sender scan: ids, sender slots and the experts' bases of up to kScanBatch
  // rows are loaded before the rows are ranked in order
  for (int it0 = a0; it0 < a1; it0 += 32 * kScanBatch) {
    int eb[kScanBatch], sb[kScanBatch], bb[kScanBatch];
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u) {
      const int a = it0 + 32 * u + lane;
      eb[u] = a < a1 ? idx[a] : 0;
      sb[u] = a < a1 ? slot[2LL * a] : -1;
    }
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u) {
      const int a = it0 + 32 * u + lane;
      const bool ok = a < a1 && eb[u] >= 0 && eb[u] < E && sb[u] >= 0;
      bb[u] = ok ? base_exp[static_cast<long long>(eb[u]) * n_chunks + c] : 0;
    }
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u) {
      if (it0 + 32 * u >= a1) break;  // warp-uniform
      const int a = it0 + 32 * u + lane;
      const int e_raw = eb[u];
      const bool valid = a < a1 && e_raw >= 0 && e_raw < E;
      const int e = valid ? e_raw : 0;
      const bool sk = valid && sb[u] >= 0;
      const int key = sk ? e : -1 - lane;
      const unsigned act = __ballot_sync(0xffffffffu, sk);
      const unsigned peers = __match_any_sync(0xffffffffu, key) & act;
      const int rank = __popc(peers & ((1u << lane) - 1u));
      int r = -1;
      if (sk) r = bb[u] + run[e] + rank;
      __syncwarp();
      if (sk && rank == __popc(peers) - 1) run[e] += __popc(peers);
      if (a < a1 && !valid) slot[2LL * a + 1] = -1;
      if (valid) {
        const bool rk = sk && r < Cr;
        slot[2LL * a + 1] = rk ? r : -1;
        if (rk) atomicAdd(&stats_kept_e[e], 1);
        else if (sk) atomicAdd(&stats_dr_e[e], 1);
        else atomicAdd(&stats_ds_e[e], 1);
      }
      __syncwarp();
    }
  }
}

// totals and maxima from the per-expert / per-pool counters (one block); with write_hist
// also the selection histogram, kept + sender-dropped + receiver-dropped of each expert
// (every assignment is exactly one of the three)
__global__ void scan_totals(int32_t* __restrict__ stats, int E, int NP, int A_total, int off_kept, int off_ds,
                            int off_dr, int off_fill, int off_hist, int write_hist) {
  __shared__ int s_kept, s_ds, s_dr, s_mp, s_me;
  if (threadIdx.x == 0) s_kept = s_ds = s_dr = s_mp = s_me = 0;
  __syncthreads();
  int k = 0, ds = 0, dr = 0, me = 0, mp = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    k += stats[off_kept + e];
    ds += stats[off_ds + e];
    dr += stats[off_dr + e];
    me = max(me, stats[off_kept + e]);
    if (write_hist) stats[off_hist + e] = stats[off_kept + e] + stats[off_ds + e] + stats[off_dr + e];
  }
  for (int p = threadIdx.x; p < NP; p += blockDim.x) mp = max(mp, stats[off_fill + p]);
  atomicAdd(&s_kept, k);
  atomicAdd(&s_ds, ds);
  atomicAdd(&s_dr, dr);
  atomicMax(&s_me, me);
  atomicMax(&s_mp, mp);
  __syncthreads();
  if (threadIdx.x == 0) {
    stats[0] = s_kept;
    stats[1] = s_ds;
    stats[2] = s_dr;
    stats[4] = s_mp;
    stats[5] = s_me;
    stats[6] = A_total;
  }
}

// ---------------------------------------------------------------------- pack / unpack

// one warp per token: read z_t once, write it into every pool row it was given
// pool of assignment (token t, expert e) across sources: source t / Ts owns the NP pools
// [source * NP, source * NP + NP), source-major
__device__ __forceinline__ int src_pool(int t, int Ts, int NP, int e, int L, int P, int W) {
  return (t / Ts) * NP + pool_of(e, L, P, W);
}

// first row of pool p: fixed-size pools at p * C_s, packed pools (dropless) at pool_off[p]
__device__ __forceinline__ long long pool_row0(int p, int Cs, const int32_t* pool_off) {
  return pool_off != nullptr ? static_cast<long long>(pool_off[p]) : static_cast<long long>(p) * Cs;
}

// first row of expert e in the expert buffers: e * C_r, or exp_off[e] (dropless)
__device__ __forceinline__ long long exp_row0(int e, int Cr, const int32_t* exp_off) {
  return exp_off != nullptr ? static_cast<long long>(exp_off[e]) : static_cast<long long>(e) * Cr;
}

__global__ void pack_kernel(const uint16_t* __restrict__ z, const int32_t* __restrict__ idx,
                            const int32_t* __restrict__ slot, int T, int k, int dl, int L, int P, int W, int Cs,
                            int E, uint16_t* __restrict__ pools, const int32_t* __restrict__ pool_off, int Ts,
                            int NPsrc) {
  // destination row of each of the token's k assignments, staged per warp in shared
  // memory (no warp shuffle inside the lane-divergent column loop)
  __shared__ long long s_dst[8][32];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int warps = blockDim.x >> 5;
  const long long row_elems = dl + 8;
  const int nvec = dl / 8;
  for (int t = blockIdx.x * warps + wib; t < T; t += gridDim.x * warps) {
    int e_j = -1, s_j = -1;
    if (lane < k) {
      e_j = idx[static_cast<long long>(t) * k + lane];
      s_j = slot[2LL * (static_cast<long long>(t) * k + lane)];
      const bool ok = s_j >= 0 && s_j < Cs && e_j >= 0 && e_j < E;
      s_dst[wib][lane] = ok ? (pool_row0(src_pool(t, Ts, NPsrc, e_j, L, P, W), Cs, pool_off) + s_j) * row_elems : -1;
    }
    __syncwarp();
    const uint4* src = reinterpret_cast<const uint4*>(z + static_cast<long long>(t) * dl);
    for (int v0 = lane; v0 < nvec; v0 += 32 * 8) {
      uint4 val[8];  // up to 8 vectors of the row in flight per lane, then k copies
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (v0 + 32 * u < nvec) val[u] = src[v0 + 32 * u];
      for (int j = 0; j < k; ++j) {
        const long long d = s_dst[wib][j];
        if (d < 0) continue;
        uint4* dst = reinterpret_cast<uint4*>(pools + d);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (v0 + 32 * u < nvec) dst[v0 + 32 * u] = val[u];
      }
    }
    if (lane < k && s_j >= 0 && s_j < Cs && e_j >= 0 && e_j < E) {
      uint16_t* dst = pools + (pool_row0(src_pool(t, Ts, NPsrc, e_j, L, P, W), Cs, pool_off) + s_j) * row_elems + dl;
      *reinterpret_cast<int4*>(dst) = make_int4(e_j, 0, 0, 0);
    }
    __syncwarp();
  }
}

// Dispatch through the copy engine.  Each warp owns three row buffers in shared memory.
// Lane 0 brings token t's latent row in with one bulk copy and sends it to each of the
// token's kept pool rows with one bulk store per row, while the next token's row is
// already loading into another buffer; lane j writes the 16-byte header of
// assignment j.  Whole-row bulk stores keep many full lines in flight per SM.  With a
// third buffer the next load waits only for the stores of two tokens back, so a warp's
// stores stream without a gap (0.195 against 0.203 ms for two buffers and 16 warps per
// SM at T=16384, top-8, latent 3072; more warps or buffers were no faster).
constexpr int kPackWarps = 8;
constexpr int kPackBufs = 3;  // row buffers per warp

__global__ void __launch_bounds__(32 * kPackWarps)
    pack_bulk_kernel(const uint16_t* __restrict__ z, const int32_t* __restrict__ idx,
                     const int32_t* __restrict__ slot, int T, int k, int dl, int L, int P, int W, int Cs, int E,
                     const int32_t* __restrict__ pool_fill, int NP, uint16_t* __restrict__ pools,
                     int32_t* __restrict__ status, const int32_t* __restrict__ pool_off, int Ts, int NPsrc) {
  extern __shared__ __align__(128) uint8_t pack_smem[];
  __shared__ uint64_t s_bar[kPackWarps][kPackBufs];
  __shared__ long long s_dst[kPackWarps][32];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const uint32_t row_bytes = static_cast<uint32_t>(dl) * 2u;
  auto buf = [&](int q) { return pack_smem + (static_cast<size_t>(wib) * kPackBufs + q) * row_bytes; };
  if (lane == 0) {
    for (int q = 0; q < kPackBufs; ++q) mbar_init(&s_bar[wib][q], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const long long row_elems = dl + 8;
  const int nw = gridDim.x * (blockDim.x >> 5);
  const int t0 = blockIdx.x * (blockDim.x >> 5) + wib;
  uint32_t armed = 0;  // per buffer: a row load is in flight
  if (lane == 0 && t0 < T) {
    mbar_arrive_expect_tx(&s_bar[wib][0], row_bytes);
    bulk_load_g2s(buf(0), z + static_cast<long long>(t0) * dl, row_bytes, &s_bar[wib][0]);
    armed = 1u;
  }
  int i = 0;
  for (int t = t0; t < T; t += nw, ++i) {
    const int b = i % kPackBufs;
    const int bn = (i + 1) % kPackBufs;
    int e_j = -1, s_j = -1;
    bool ok_j = false;
    if (lane < k) {
      e_j = idx[static_cast<long long>(t) * k + lane];
      s_j = slot[2LL * (static_cast<long long>(t) * k + lane)];
      ok_j = s_j >= 0 && s_j < Cs && e_j >= 0 && e_j < E;
      s_dst[wib][lane] = ok_j ? (pool_row0(src_pool(t, Ts, NPsrc, e_j, L, P, W), Cs, pool_off) + s_j) * row_elems : -1;
    }
    __syncwarp();
    bool got = true;
    if (lane == 0) {
      const int tn = t + nw;
      if (tn < T) {
        // the stores of the token that last used the next buffer (kPackBufs - 1 tokens
        // ago) have read it
        bulk_wait_read<kPackBufs - 2>();
        mbar_arrive_expect_tx(&s_bar[wib][bn], row_bytes);
        bulk_load_g2s(buf(bn), z + static_cast<long long>(tn) * dl, row_bytes, &s_bar[wib][bn]);
        armed |= 1u << bn;
      }
      got = mbar_wait(&s_bar[wib][b], static_cast<uint32_t>((i / kPackBufs) & 1), nullptr);
      armed &= ~(1u << b);
      if (got) {
        fence_proxy_async_shared();
        for (int j = 0; j < k; ++j) {
          const long long d = s_dst[wib][j];
          if (d >= 0) bulk_store_s2g(pools + d, buf(b), row_bytes);
        }
        bulk_commit();
      }
    }
    got = __shfl_sync(0xffffffffu, got, 0);
    if (!got) {
      if (lane == 0) {
        record_status_i32(status, MOE_ERR_TIMEOUT);
        // let a row load still in flight land before the warp leaves
        if (armed & (1u << bn)) mbar_wait(&s_bar[wib][bn], static_cast<uint32_t>(((i + 1) / kPackBufs) & 1), nullptr);
      }
      break;
    }
    if (ok_j) *reinterpret_cast<int4*>(pools + s_dst[wib][lane] + dl) = make_int4(e_j, 0, 0, 0);
    __syncwarp();
  }
  // header -1 for the rows of each pool past its fill (slots below the fill are dense);
  // packed pools (dropless) have no such rows
  const long long n_rows = pool_off != nullptr ? 0 : static_cast<long long>(NP) * Cs;
  for (long long rr = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; rr < n_rows;
       rr += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int pl = static_cast<int>(rr / Cs);
    if (static_cast<int>(rr - static_cast<long long>(pl) * Cs) >= pool_fill[pl])
      *reinterpret_cast<int4*>(pools + rr * row_elems + dl) = make_int4(-1, 0, 0, 0);
  }
  if (lane == 0) bulk_wait_all();
}

// header -1 for the rows of each pool past its fill
__global__ void pack_empty_headers(const int32_t* __restrict__ pool_fill, int NP, int Cs, int dl,
                                   uint16_t* __restrict__ pools) {
  const long long row_elems = dl + 8;
  const long long total = static_cast<long long>(NP) * Cs;
  for (long long r = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; r < total;
       r += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(r / Cs);
    const int s = static_cast<int>(r % Cs);
    if (s >= pool_fill[p]) *reinterpret_cast<int4*>(pools + r * row_elems + dl) = make_int4(-1, 0, 0, 0);
  }
}

// receiver, pass 1: one block per pool.  Rows are visited in pool order in tiles of the
// block size; a row whose packed id names local expert q of this pool gets the next slot
// of q.  The first C_r rows of each expert are mapped to their receive-buffer row
// (e * C_r + slot) in row_map; other rows map to -1.
__global__ void unpack_rank_kernel(const uint16_t* __restrict__ pools, int Cs, int Cr, int dl, int L, int P, int W,
                                   int32_t* __restrict__ row_map, int32_t* __restrict__ rows_out,
                                   int32_t* __restrict__ status, const int32_t* __restrict__ pool_off,
                                   const int32_t* __restrict__ pool_fill, int S, int id_base) {
  constexpr int kTile = 256;
  __shared__ int s_warp_cnt[kTile / 32][32];
  __shared__ int s_run[32];
  const int pool = blockIdx.x;  // (destination, wave); its pools from every source, in order
  const int NPsrc = gridDim.x;
  const int dest = pool / W, wave = pool % W;
  const int e_first = dest * L + wave * P;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long row_elems = dl + 8;
  if (threadIdx.x < 32) s_run[threadIdx.x] = 0;
  __syncthreads();
  // packed pools (dropless): this pool's rows are the pool_fill[pool] rows at pool_off[pool],
  // the row map holds the receiver slot and every row is kept
  const bool packed = pool_off != nullptr;
  for (int src = 0; src < S; ++src) {
    const int qpool = src * NPsrc + pool;
    const long long prow0 = pool_row0(qpool, Cs, pool_off);
    const int nrows = packed ? pool_fill[qpool] : Cs;
    const uint16_t* pbase = pools + prow0 * row_elems;
    for (int r0 = 0; r0 < nrows; r0 += kTile) {
      const int r = r0 + threadIdx.x;
      int q = -1;
      if (r < nrows) {
        // packed ids are global; a receiver of experts [id_base, ...) numbers them from 0
        const int eg = *reinterpret_cast<const int*>(pbase + r * row_elems + dl);
        const int e = eg >= 0 ? eg - id_base : -1;
        if (eg >= 0) {
          if (e >= e_first && e < e_first + P) q = e - e_first;
          else atomicCAS(status, 0, MOE_ERR_INVALID_ARG);  // an id this pool cannot hold
        }
      }
      // rank of this row among the tile's rows of the same local expert, in row order
      int rank = 0;
      for (int qq = 0; qq < P; ++qq) {
        const unsigned m = __ballot_sync(0xffffffffu, q == qq);
        if (q == qq) rank = __popc(m & ((1u << lane) - 1u));
        if (lane == 0) s_warp_cnt[warp][qq] = __popc(m);
      }
      __syncthreads();
      int slot = -1;
      if (q >= 0) {
        int before = s_run[q];
        for (int w = 0; w < warp; ++w) before += s_warp_cnt[w][q];
        slot = before + rank;
      }
      if (r < nrows)
        row_map[prow0 + r] = packed ? slot : ((slot >= 0 && slot < Cr) ? (e_first + q) * Cr + slot : -1);
      __syncthreads();
      if (threadIdx.x < P) {
        int tot = 0;
        for (int w = 0; w < kTile / 32; ++w) tot += s_warp_cnt[w][threadIdx.x];
        s_run[threadIdx.x] += tot;
      }
      __syncthreads();
    }
  }  // sources
  if (threadIdx.x < P) rows_out[e_first + threadIdx.x] = packed ? s_run[threadIdx.x] : min(s_run[threadIdx.x], Cr);
}

// receiver, pass 2: one warp per pool row, up to 8 vectors per lane in flight
__global__ void unpack_copy_kernel(const uint16_t* __restrict__ pools, const int32_t* __restrict__ row_map,
                                   long long n_rows, int dl, uint16_t* __restrict__ xe,
                                   const int32_t* __restrict__ exp_off, int E) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const long long row_elems = dl + 8;
  const int nvec = dl / 8;
  for (long long r = static_cast<long long>(blockIdx.x) * warps + (threadIdx.x >> 5); r < n_rows;
       r += static_cast<long long>(gridDim.x) * warps) {
    long long d = row_map[r];
    if (d < 0) continue;
    if (exp_off != nullptr) {  // packed buffers: the row map holds the slot within the expert
      const int e = *reinterpret_cast<const int*>(pools + r * row_elems + dl);
      if (e < 0 || e >= E) continue;
      d += exp_off[e];
    }
    const uint4* src = reinterpret_cast<const uint4*>(pools + r * row_elems);
    uint4* dst = reinterpret_cast<uint4*>(xe + d * dl);
    for (int v0 = lane; v0 < nvec; v0 += 32 * 8) {
      uint4 val[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (v0 + 32 * u < nvec) val[u] = src[v0 + 32 * u];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (v0 + 32 * u < nvec) dst[v0 + 32 * u] = val[u];
    }
  }
}

// Rows between pool positions and expert rows under expert parallelism, one warp per pool
// row r of a receiver (its G sources' pools, in order), map[r] = expert row or -1:
//   to_pools: out[r] = in[map[r]] (expert row sent back to its pool position), zeros for a
//             receiver-dropped row; rows whose pool header says empty are not written
//             (their source never reads them)
//   else:     out[map[r]] = in[r] (a received row placed in its expert's buffer)
// Rows are `width` bf16 wide; pool-side rows have stride ld_pool, expert rows `width`.
__global__ void map_rows_kernel(const uint16_t* __restrict__ in, uint16_t* __restrict__ out,
                                const int32_t* __restrict__ map, const uint16_t* __restrict__ hdr_pools,
                                int hdr_ld, int hdr_col, long long n_rows, int width, long long ld_pool,
                                int to_pools) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int nvec = width / 8;
  for (long long r = static_cast<long long>(blockIdx.x) * warps + (threadIdx.x >> 5); r < n_rows;
       r += static_cast<long long>(gridDim.x) * warps) {
    const long long d = map[r];
    if (to_pools) {
      if (*reinterpret_cast<const int*>(hdr_pools + r * hdr_ld + hdr_col) < 0) continue;  // empty pool row
      uint4* dst = reinterpret_cast<uint4*>(out + r * ld_pool);
      const uint4* src = reinterpret_cast<const uint4*>(in + (d >= 0 ? d : 0) * width);
      for (int v = lane; v < nvec; v += 32) dst[v] = d >= 0 ? src[v] : make_uint4(0, 0, 0, 0);
    } else {
      if (d < 0) continue;
      const uint4* src = reinterpret_cast<const uint4*>(in + r * ld_pool);
      uint4* dst = reinterpret_cast<uint4*>(out + d * width);
      for (int v = lane; v < nvec; v += 32) dst[v] = src[v];
    }
  }
}

// rows [n_e, min(round_up(n_e, 128), C_r)) of each expert's buffer become zero, so that
// the GEMM tiles that cover them read zeros
__global__ void zero_tail_rows_kernel(uint16_t* __restrict__ buf, long long width, int Cr,
                                      const int32_t* __restrict__ rows, const int32_t* __restrict__ exp_off) {
  const int e = blockIdx.y;
  const int n = rows[e];
  // packed buffers (dropless): the expert's region is exactly round_up(n, 128) rows
  const int end = exp_off != nullptr ? ((n + 127) / 128) * 128 : min(((n + 127) / 128) * 128, Cr);
  const long long nvec = width / 8;
  const long long total = static_cast<long long>(end - n) * nvec;
  uint4* base = reinterpret_cast<uint4*>(buf + (exp_row0(e, Cr, exp_off) + n) * width);
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    base[i] = make_uint4(0, 0, 0, 0);
}

// ---------------------------------------------------------------------- combine and its backward

// Where the expert row of an assignment lives.  Receiver side (one GPU): expert e's rows
// start at e * C_r (or exp_off[e], packed) and the row is the receiver slot.  Source side
// under expert parallelism: the rows the receivers sent back sit in pool order, row
// pool(e) * C_s + sender slot, and a receiver-dropped row comes back as zeros.
struct RowAddr {
  int Cr;
  const int32_t* exp_off;
  int by_pool;
  int Cs, L, P, W;
};

__device__ __forceinline__ long long row_of(const RowAddr& ra, int e, const int32_t* slot_pair) {
  if (ra.by_pool) {
    const int s = slot_pair[0];
    return (s >= 0 && s < ra.Cs) ? static_cast<long long>(pool_of(e, ra.L, ra.P, ra.W)) * ra.Cs + s : -1;
  }
  const int rs = slot_pair[1];
  return (rs >= 0 && rs < ra.Cr) ? exp_row0(e, ra.Cr, ra.exp_off) + rs : -1;
}

__device__ __forceinline__ void acc8(float (&acc)[8], const uint4& v, float g) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] = fmaf(g, __uint_as_float(w[i] << 16), acc[2 * i]);
    acc[2 * i + 1] = fmaf(g, __uint_as_float(w[i] & 0xFFFF0000u), acc[2 * i + 1]);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&a)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a[2 * i], a[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&v);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// r_t = sum_j g_tj Y[row_tj] over the kept assignments, fp32 in j order.  Per pass a lane
// covers kCombVpl 16-byte vectors of the row and loads them from eight expert rows at
// once (rows past k or dropped read as zero), so a warp keeps 8 x kCombVpl x 512 bytes
// of loads in flight instead of walking the rows one after another.
constexpr int kCombVpl = 2;
constexpr int kCombRows = 8;

__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ ye, const float* __restrict__ gate,
                               const int32_t* __restrict__ idx, const int32_t* __restrict__ slot, int T, int k,
                               int dl, int E, uint16_t* __restrict__ r, const RowAddr ra) {
  __shared__ long long s_row[8][32];
  __shared__ float s_g[8][32];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int warps = blockDim.x >> 5;
  const int nvec = dl / 8;
  for (int t = blockIdx.x * warps + wib; t < T; t += gridDim.x * warps) {
    if (lane < k) {
      const long long a = static_cast<long long>(t) * k + lane;
      const int e = idx[a];
      const long long row = (e >= 0 && e < E) ? row_of(ra, e, slot + 2 * a) : -1;
      s_row[wib][lane] = row;
      s_g[wib][lane] = row >= 0 ? gate[a] : 0.0f;
    }
    __syncwarp();
    for (int v0 = lane; v0 < nvec; v0 += 32 * kCombVpl) {
      float acc[kCombVpl][8];
#pragma unroll
      for (int u = 0; u < kCombVpl; ++u)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
      for (int j0 = 0; j0 < k; j0 += kCombRows) {
        uint4 val[kCombRows][kCombVpl];
#pragma unroll
        for (int jj = 0; jj < kCombRows; ++jj) {
          const int j = j0 + jj;
          const long long rj = j < k ? s_row[wib][j] : -1;
          const uint4* yrow = reinterpret_cast<const uint4*>(ye + (rj >= 0 ? rj : 0) * dl);
#pragma unroll
          for (int u = 0; u < kCombVpl; ++u) {
            const int v = v0 + 32 * u;
            val[jj][u] = (rj >= 0 && v < nvec) ? yrow[v] : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int jj = 0; jj < kCombRows; ++jj) {
          const int j = j0 + jj;
          if (j >= k) break;
          const float g = s_g[wib][j];
#pragma unroll
          for (int u = 0; u < kCombVpl; ++u) acc8(acc[u], val[jj][u], g);
        }
      }
      uint4* out = reinterpret_cast<uint4*>(r + static_cast<long long>(t) * dl);
#pragma unroll
      for (int u = 0; u < kCombVpl; ++u)
        if (v0 + 32 * u < nvec) out[v0 + 32 * u] = pack8(acc[u]);
    }
    __syncwarp();
  }
}

// dY[row_tj] = g_tj dr_t on kept rows, dg_tj = <dr_t, Y[row_tj]>.  Per pass a lane holds
// kCombVpl vectors of dr_t and loads the matching vectors of eight expert rows at once;
// the eight partial dot products stay in registers until the row is done.
__global__ void __launch_bounds__(256) combine_bwd_kernel(const uint16_t* __restrict__ dr, const uint16_t* __restrict__ ye,
                                   const float* __restrict__ gate, const int32_t* __restrict__ idx,
                                   const int32_t* __restrict__ slot, int T, int k, int dl, int E,
                                   uint16_t* __restrict__ dye, float* __restrict__ dg, const RowAddr ra) {
  __shared__ long long s_row[8][32];
  __shared__ float s_g[8][32];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int warps = blockDim.x >> 5;
  const int nvec = dl / 8;
  for (int t = blockIdx.x * warps + wib; t < T; t += gridDim.x * warps) {
    if (lane < k) {
      const long long a = static_cast<long long>(t) * k + lane;
      const int e = idx[a];
      const long long row = (e >= 0 && e < E) ? row_of(ra, e, slot + 2 * a) : -1;
      s_row[wib][lane] = row;
      s_g[wib][lane] = row >= 0 ? gate[a] : 0.0f;
    }
    __syncwarp();
    const uint4* drow = reinterpret_cast<const uint4*>(dr + static_cast<long long>(t) * dl);
    for (int j0 = 0; j0 < k; j0 += kCombRows) {
      float dot[kCombRows];
#pragma unroll
      for (int jj = 0; jj < kCombRows; ++jj) dot[jj] = 0.0f;
      for (int v0 = lane; v0 < nvec; v0 += 32 * kCombVpl) {
        uint4 d[kCombVpl], y[kCombRows][kCombVpl];
#pragma unroll
        for (int u = 0; u < kCombVpl; ++u) {
          const int v = v0 + 32 * u;
          d[u] = v < nvec ? drow[v] : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int jj = 0; jj < kCombRows; ++jj) {
          const int j = j0 + jj;
          const long long rj = j < k ? s_row[wib][j] : -1;
          const uint4* yrow = reinterpret_cast<const uint4*>(ye + (rj >= 0 ? rj : 0) * dl);
#pragma unroll
          for (int u = 0; u < kCombVpl; ++u) {
            const int v = v0 + 32 * u;
            y[jj][u] = (rj >= 0 && v < nvec) ? yrow[v] : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int jj = 0; jj < kCombRows; ++jj) {
          const int j = j0 + jj;
          const long long rj = j < k ? s_row[wib][j] : -1;
          if (rj < 0) continue;
          const float g = s_g[wib][j];
          uint4* out = reinterpret_cast<uint4*>(dye + rj * dl);
#pragma unroll
          for (int u = 0; u < kCombVpl; ++u) {
            const int v = v0 + 32 * u;
            if (v >= nvec) continue;
            const uint32_t dw[4] = {d[u].x, d[u].y, d[u].z, d[u].w};
            const uint32_t yw[4] = {y[jj][u].x, y[jj][u].y, y[jj][u].z, y[jj][u].w};
            float o[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float d0 = __uint_as_float(dw[i] << 16), d1 = __uint_as_float(dw[i] & 0xFFFF0000u);
              const float y0 = __uint_as_float(yw[i] << 16), y1 = __uint_as_float(yw[i] & 0xFFFF0000u);
              dot[jj] = fmaf(d0, y0, dot[jj]);
              dot[jj] = fmaf(d1, y1, dot[jj]);
              o[2 * i] = g * d0;
              o[2 * i + 1] = g * d1;
            }
            out[v] = pack8(o);
          }
        }
      }
#pragma unroll
      for (int jj = 0; jj < kCombRows; ++jj) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dot[jj] += __shfl_xor_sync(0xffffffffu, dot[jj], off);
      }
      if (lane < kCombRows && j0 + lane < k) {
        float mine = 0.0f;
#pragma unroll
        for (int jj = 0; jj < kCombRows; ++jj)
          if (jj == lane) mine = dot[jj];
        dg[static_cast<long long>(t) * k + j0 + lane] = s_row[wib][j0 + lane] >= 0 ? mine : 0.0f;
      }
    }
    __syncwarp();
  }
}

// dz_routed_t = sum_j kept dX[e_tj][rslot_tj]; dlogits_t = softmax backward over the
// chosen experts, zero elsewhere
__global__ void undispatch_kernel(const uint16_t* __restrict__ dxe, const float* __restrict__ gate,
                                  const float* __restrict__ dg, const int32_t* __restrict__ idx,
                                  const int32_t* __restrict__ slot, int T, int k, int dl, int E,
                                  float* __restrict__ dz, uint16_t* __restrict__ dlogits, const RowAddr ra) {
  __shared__ long long s_row[8][32];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int warps = blockDim.x >> 5;
  const int nvec = dl / 8;
  for (int t = blockIdx.x * warps + wib; t < T; t += gridDim.x * warps) {
    float g_j = 0.0f, dg_j = 0.0f;
    int e_j = -1;
    if (lane < k) {
      const long long a = static_cast<long long>(t) * k + lane;
      e_j = idx[a];
      g_j = gate[a];
      dg_j = dg[a];
      if (e_j < 0 || e_j >= E) e_j = -1;
      s_row[wib][lane] = e_j >= 0 ? row_of(ra, e_j, slot + 2 * a) : -1;
    }
    __syncwarp();
    // as in the combine: the matching vectors of up to kCombRows rows are loaded at once,
    // then summed in j order (rows of dropped assignments are skipped)
    for (int v0 = lane; v0 < nvec; v0 += 32 * kCombVpl) {
      float acc[kCombVpl][8];
#pragma unroll
      for (int u = 0; u < kCombVpl; ++u)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
      for (int j0 = 0; j0 < k; j0 += kCombRows) {
        uint4 val[kCombRows][kCombVpl];
#pragma unroll
        for (int jj = 0; jj < kCombRows; ++jj) {
          const int j = j0 + jj;
          const long long rj = j < k ? s_row[wib][j] : -1;
          const uint4* xrow = reinterpret_cast<const uint4*>(dxe + (rj >= 0 ? rj : 0) * dl);
#pragma unroll
          for (int u = 0; u < kCombVpl; ++u) {
            const int v = v0 + 32 * u;
            val[jj][u] = (rj >= 0 && v < nvec) ? xrow[v] : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int jj = 0; jj < kCombRows; ++jj) {
          const int j = j0 + jj;
          if (j >= k) break;
          if (s_row[wib][j] < 0) continue;
#pragma unroll
          for (int u = 0; u < kCombVpl; ++u) acc8(acc[u], val[jj][u], 1.0f);
        }
      }
#pragma unroll
      for (int u = 0; u < kCombVpl; ++u) {
        const int v = v0 + 32 * u;
        if (v < nvec) {
          float4* o = reinterpret_cast<float4*>(dz + static_cast<long long>(t) * dl + 8 * v);
          o[0] = make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
          o[1] = make_float4(acc[u][4], acc[u][5], acc[u][6], acc[u][7]);
        }
      }
    }
    // softmax backward: dl_j = g_j (dg_j - sum_i g_i dg_i)
    float s = lane < k ? g_j * dg_j : 0.0f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    uint16_t* drow = dlogits + static_cast<long long>(t) * E;
    for (int e = lane; e < E; e += 32) drow[e] = 0;
    __syncwarp();
    if (lane < k && e_j >= 0) {
      const float d = g_j * (dg_j - s);
      __nv_bfloat16 b = __float2bfloat16_rn(d);
      drow[e_j] = *reinterpret_cast<uint16_t*>(&b);
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------- bias step

__global__ void bias_update_kernel(const int32_t* __restrict__ hist, float* __restrict__ bias, int E, long long Tk,
                                   float step) {
  __shared__ int warp_sum[32];
  const int e = threadIdx.x;
  int sgn = 0;
  if (e < E) {
    const long long load = static_cast<long long>(E) * hist[e];
    sgn = (Tk > load) - (Tk < load);
  }
  int s = sgn;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = s;
  __syncthreads();
  int total = 0;
  for (int w = 0; w < (blockDim.x + 31) / 32; ++w) total += warp_sum[w];
  if (e < E) {
    const float mean = __fdiv_rn(static_cast<float>(total), static_cast<float>(E));
    const float delta = __fsub_rn(static_cast<float>(sgn), mean);
    bias[e] = __fadd_rn(bias[e], __fmul_rn(step, delta));
  }
}

int blocks_for(long long work, int per_block) {
  long long b = (work + per_block - 1) / per_block;
  const long long cap = 8LL * device_sm_count();
  if (b > cap) b = cap;
  return static_cast<int>(b < 1 ? 1 : b);
}

}  // namespace

// off[i] = sum over j < i of round_up(counts[j], align), for i = 0..n; one block of 1024
// threads walking the counts 1024 at a time (negative counts read as zero)
__global__ void __launch_bounds__(1024) offsets_kernel(const int32_t* __restrict__ counts, int n, int align,
                                                       int32_t* __restrict__ off) {
  __shared__ int s_warp[32];
  __shared__ int s_carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + threadIdx.x;
    int v = 0;
    if (i < n) {
      const int c = counts[i] > 0 ? counts[i] : 0;
      v = (c + align - 1) / align * align;
    }
    int incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += u;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = s_warp[lane];
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, w, d);
        if (lane >= d) w += u;
      }
      s_warp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int before = s_carry + (warp > 0 ? s_warp[warp - 1] : 0);
    if (i < n) off[i] = before + incl - v;
    __syncthreads();
    if (threadIdx.x == 1023) s_carry = before + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) off[n] = s_carry;
}

// out[i] = sum over s of part[s][i] (float32, s in order): the K slices of a split weight
// gradient
__global__ void sum_partials_kernel(const float4* __restrict__ part, int S, long long n4, float4* __restrict__ out) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float4 a = part[i];
    for (int s = 1; s < S; ++s) {
      const float4 b = part[s * n4 + i];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    out[i] = a;
  }
}

// ====================================================================== launchers

moe_status_t launch_route(const Geo& g, const float* logits, const float* bias, int32_t* idx, float* gate,
                          int32_t* hist, int32_t* nan_count, cudaStream_t st) {
  if (g.T == 0) return MOE_OK;
  const int warps = 8;
  const int vpl = (g.E + 31) / 32;
  // persistent: as many blocks as fit at once, each warp walking several tokens
#define MOE_ROUTE(V)                                                                                       \
  if (vpl <= V) {                                                                                          \
    int per_sm = 1;                                                                                        \
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_topk_kernel<V>, 32 * warps, 0) !=     \
            cudaSuccess ||                                                                                 \
        per_sm < 1)                                                                                        \
      per_sm = 1;                                                                                          \
    const int grid = static_cast<int>(                                                                     \
        std::min<long long>(blocks_for(g.T, warps), static_cast<long long>(device_sm_count()) * per_sm));  \
    route_topk_kernel<V><<<grid, 32 * warps, 0, st>>>(logits, bias, g.T, g.E, g.k, idx, gate, hist, nan_count); \
    count_launch();                                                                                          \
    return cuda_check(cudaGetLastError(), "route_topk");                                                    \
  }
  MOE_ROUTE(1)
  MOE_ROUTE(2)
  MOE_ROUTE(4)
  MOE_ROUTE(8)
  MOE_ROUTE(12)
  MOE_ROUTE(16)
  MOE_ROUTE(32)
#undef MOE_ROUTE
  return fail(MOE_ERR_UNSUPPORTED, "too many experts for the router kernel");
}

size_t scan_scratch_ints(const Geo& g) {
  return static_cast<size_t>(g.n_chunks) * (g.NP + g.E) + g.NPS;
}

moe_status_t launch_slot_scan(const Geo& g, const int32_t* idx, int32_t* slot, int32_t* stats, int32_t* scratch,
                              cudaStream_t st, bool write_hist) {
  const int A = g.T * g.k;
  const int chunk_assign = kScanTokensPerChunk * g.k;
  int32_t* cnt_pool = scratch;                                        // [NP][n_chunks]
  int32_t* cnt_exp = scratch + static_cast<size_t>(g.n_chunks) * g.NP;  // [E][n_chunks]
  int32_t* pool_tot = cnt_exp + static_cast<size_t>(g.n_chunks) * g.E;  // [S][NP]
  // counters of this call start at zero (hist is left to the router)
  cudaError_t e = cudaMemsetAsync(stats + stats_kept_e(g), 0, sizeof(int32_t) * 3 * g.E, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(stats, 0, sizeof(int32_t) * 3, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(stats + 4, 0, sizeof(int32_t) * 3, st);
  if (e != cudaSuccess) return cuda_check(e, "slot scan memset");
  if (A == 0) {
    e = cudaMemsetAsync(stats + stats_pool_fill(g), 0, sizeof(int32_t) * g.NPS, st);
    if (e == cudaSuccess && write_hist) e = cudaMemsetAsync(stats + stats_hist(g), 0, sizeof(int32_t) * g.E, st);
    return cuda_check(e, "slot scan memset");
  }
  scan_count_pools<<<g.n_chunks, 256, g.NP * sizeof(int), st>>>(idx, A, chunk_assign, g.n_chunks, g.L, g.P, g.W,
                                                                 g.NP, g.E, cnt_pool);
  // sender slots count per (source, pool): the scan restarts at each source's first chunk
  scan_rows<<<g.NP, 256, 0, st>>>(cnt_pool, g.n_chunks, pool_tot, g.Cs, stats + stats_pool_fill(g),
                                  g.n_chunks / g.S);
  const int wpb = 4;
  const int grid = (g.n_chunks + wpb - 1) / wpb;
  scan_sender_slots<<<grid, 32 * wpb, wpb * (g.NP + g.E) * sizeof(int), st>>>(
      idx, A, chunk_assign, g.n_chunks, g.L, g.P, g.W, g.NP, g.E, g.Cs, cnt_pool, slot, cnt_exp, stats + 3);
  scan_rows<<<g.E, 256, 0, st>>>(cnt_exp, g.n_chunks, nullptr, 0, nullptr, g.n_chunks);
  scan_receiver_slots<<<grid, 32 * wpb, wpb * g.E * sizeof(int), st>>>(
      idx, A, chunk_assign, g.n_chunks, g.E, g.Cr, cnt_exp, slot, stats + stats_kept_e(g), stats + stats_ds_e(g),
      stats + stats_dr_e(g));
  scan_totals<<<1, 256, 0, st>>>(stats, g.E, g.NPS, A, stats_kept_e(g), stats_ds_e(g), stats_dr_e(g),
                                 stats_pool_fill(g), stats_hist(g), write_hist ? 1 : 0);
  count_launch(6);
  return cuda_check(cudaGetLastError(), "slot scan");
}

moe_status_t launch_pack(const Geo& g, const uint16_t* z, const int32_t* idx, const int32_t* slot,
                         int32_t* stats, uint16_t* pools, cudaStream_t st, const int32_t* pool_off) {
  if (g.T > 0) {
    // kPackBufs row buffers per warp; rows too wide for that take the register path
    const size_t smem = static_cast<size_t>(kPackWarps) * kPackBufs * g.dl * 2;
    if (g.k <= 32 && smem <= 200 * 1024) {
      static std::atomic<uint64_t> attr_done{0};  // one bit per device
      const moe_status_t r =
          ensure_max_smem(reinterpret_cast<const void*>(pack_bulk_kernel), 200 * 1024, attr_done, "pack");
      if (r != MOE_OK) return r;
      int per_sm = 1;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pack_bulk_kernel, 32 * kPackWarps, smem) !=
              cudaSuccess ||
          per_sm < 1)
        per_sm = 1;
      const int grid = static_cast<int>(std::min<long long>((g.T + kPackWarps - 1) / kPackWarps,
                                                            static_cast<long long>(device_sm_count()) * per_sm));
      pack_bulk_kernel<<<grid, 32 * kPackWarps, smem, st>>>(z, idx, slot, g.T, g.k, g.dl, g.L, g.P, g.W, g.Cs, g.E,
                                                            stats + stats_pool_fill(g), g.NPS, pools, stats + 3,
                                                            pool_off, g.Ts, g.NP);
      count_launch();
      return cuda_check(cudaGetLastError(), "pack");
    } else {
      const int warps = 8;
      pack_kernel<<<blocks_for(g.T, warps), 32 * warps, 0, st>>>(z, idx, slot, g.T, g.k, g.dl, g.L, g.P, g.W, g.Cs,
                                                                 g.E, pools, pool_off, g.Ts, g.NP);
    }
    count_launch();
  }
  const long long rows = pool_off != nullptr ? 0 : static_cast<long long>(g.NPS) * g.Cs;
  if (rows > 0)
  {
    pack_empty_headers<<<blocks_for(rows, 256), 256, 0, st>>>(stats + stats_pool_fill(g), g.NPS, g.Cs, g.dl, pools);
    count_launch();
  }
  return cuda_check(cudaGetLastError(), "pack");
}

size_t unpack_scratch_ints(const Geo& g) { return static_cast<size_t>(g.pool_rows); }

moe_status_t launch_offsets(const int32_t* counts, int n, int align, int32_t* off, cudaStream_t st) {
  if (n < 0 || align < 1) return fail(MOE_ERR_INVALID_ARG, "offsets need n >= 0 and align >= 1");
  offsets_kernel<<<1, 1024, 0, st>>>(counts, n, align, off);
  count_launch();
  return cuda_check(cudaGetLastError(), "offsets");
}

moe_status_t launch_unpack(const Geo& g, const uint16_t* pools, uint16_t* xe, int32_t* rows, int32_t* row_map,
                           int32_t* status, cudaStream_t st, const int32_t* pool_off, const int32_t* pool_fill,
                           int32_t* exp_off, int id_base) {
  if (g.P > 32) return fail(MOE_ERR_UNSUPPORTED, "more than 32 experts per wave");
  const bool packed = pool_off != nullptr;
  if (packed && (pool_fill == nullptr || exp_off == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "packed pools need their fills and the expert offsets");
  unpack_rank_kernel<<<g.NP, 256, 0, st>>>(pools, g.Cs, g.Cr, g.dl, g.L, g.P, g.W, row_map, rows, status, pool_off,
                                           pool_fill, g.S, id_base);
  count_launch();
  if (packed) MOE_TRY_K(launch_offsets(rows, g.E, 128, exp_off, st));
  const long long n_rows = g.pool_rows;
  const int warps = 8;
  unpack_copy_kernel<<<blocks_for(n_rows, warps), 32 * warps, 0, st>>>(pools, row_map, n_rows, g.dl, xe,
                                                                       packed ? exp_off : nullptr, g.E);
  count_launch();
  return cuda_check(cudaGetLastError(), "unpack");
}

moe_status_t launch_map_rows(const uint16_t* in, uint16_t* out, const int32_t* map, const uint16_t* hdr_pools,
                             int hdr_ld, int hdr_col, long long n_rows, int width, long long ld_pool, bool to_pools,
                             cudaStream_t st) {
  if (n_rows <= 0) return MOE_OK;
  if (width % 8 != 0 || ld_pool % 8 != 0) return fail(MOE_ERR_INVALID_ARG, "row mover needs 16-byte rows");
  const int warps = 8;
  map_rows_kernel<<<blocks_for(n_rows, warps), 32 * warps, 0, st>>>(in, out, map, hdr_pools, hdr_ld, hdr_col, n_rows,
                                                                    width, ld_pool, to_pools ? 1 : 0);
  count_launch();
  return cuda_check(cudaGetLastError(), "map rows");
}

moe_status_t launch_zero_tail_rows(const Geo& g, uint16_t* buf, int64_t width, const int32_t* rows,
                                   cudaStream_t st, const int32_t* exp_off) {
  dim3 grid(4, g.E);
  zero_tail_rows_kernel<<<grid, 256, 0, st>>>(buf, width, g.Cr, rows, exp_off);
  count_launch();
  return cuda_check(cudaGetLastError(), "zero tail rows");
}

namespace {
RowAddr row_addr(const Geo& g, const int32_t* exp_off, bool by_pool) {
  RowAddr ra;
  ra.Cr = g.Cr;
  ra.exp_off = exp_off;
  ra.by_pool = by_pool ? 1 : 0;
  ra.Cs = g.Cs;
  ra.L = g.L;
  ra.P = g.P;
  ra.W = g.W;
  return ra;
}
}  // namespace

moe_status_t launch_combine(const Geo& g, const uint16_t* ye, const float* gate, const int32_t* idx,
                            const int32_t* slot, uint16_t* r, cudaStream_t st, const int32_t* exp_off,
                            bool by_pool) {
  if (g.T == 0) return MOE_OK;
  const int warps = 8;
  combine_kernel<<<blocks_for(g.T, warps), 32 * warps, 0, st>>>(ye, gate, idx, slot, g.T, g.k, g.dl, g.E, r,
                                                                row_addr(g, exp_off, by_pool));
  count_launch();
  return cuda_check(cudaGetLastError(), "combine");
}

moe_status_t launch_combine_bwd(const Geo& g, const uint16_t* dr, const uint16_t* ye, const float* gate,
                                const int32_t* idx, const int32_t* slot, uint16_t* dye, float* dg,
                                cudaStream_t st, const int32_t* exp_off, bool by_pool) {
  if (g.T == 0) return MOE_OK;
  const int warps = 8;
  combine_bwd_kernel<<<blocks_for(g.T, warps), 32 * warps, 0, st>>>(dr, ye, gate, idx, slot, g.T, g.k, g.dl,
                                                                    g.E, dye, dg, row_addr(g, exp_off, by_pool));
  count_launch();
  return cuda_check(cudaGetLastError(), "combine_bwd");
}

moe_status_t launch_undispatch(const Geo& g, const uint16_t* dxe, const float* gate, const float* dg,
                               const int32_t* idx, const int32_t* slot, float* dz_routed, uint16_t* dlogits,
                               cudaStream_t st, const int32_t* exp_off, bool by_pool) {
  if (g.T == 0) return MOE_OK;
  const int warps = 8;
  undispatch_kernel<<<blocks_for(g.T, warps), 32 * warps, 0, st>>>(dxe, gate, dg, idx, slot, g.T, g.k, g.dl,
                                                                   g.E, dz_routed, dlogits,
                                                                   row_addr(g, exp_off, by_pool));
  count_launch();
  return cuda_check(cudaGetLastError(), "undispatch");
}

moe_status_t launch_sum_partials(const float* part, int S, long long n, float* out, cudaStream_t st) {
  if (n <= 0) return MOE_OK;
  if (n % 4 != 0) return fail(MOE_ERR_UNSUPPORTED, "partial sums need a multiple of 4 elements");
  const long long n4 = n / 4;
  const int grid = static_cast<int>(std::min<long long>((n4 + 255) / 256, 4LL * device_sm_count()));
  sum_partials_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const float4*>(part), S, n4, reinterpret_cast<float4*>(out));
  count_launch();
  return cuda_check(cudaGetLastError(), "sum partials");
}

moe_status_t launch_bias_update(const Geo& g, const int32_t* hist, float* bias, float step, cudaStream_t st) {
  const int threads = ((g.E + 31) / 32) * 32;
  bias_update_kernel<<<1, threads, 0, st>>>(hist, bias, g.E, static_cast<long long>(g.T) * g.k, step);
  count_launch();
  return cuda_check(cudaGetLastError(), "bias_update");
}

}  // namespace moe
