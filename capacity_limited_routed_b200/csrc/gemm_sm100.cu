// gemm_sm100.cu -- persistent tcgen05 GEMM for sm_100a: TMA -> shared memory -> tcgen05.mma ->
// TMEM accumulators -> fused epilogues.
//
// These are the dense contractions of the MoE block: the latent down- and
// up-projections, the router, the grouped SwiGLU experts and the shared experts,
// with their transposed forms for the backward pass ("Marin начинает открытое
// обучение MoE-модели с 535 млрд параметров", §2; "Marin 535B-A23B：一场完全公开的前沿
// MoE 训练直播", §2.2).
//
// Structure (one CTA per SM, 192 threads):
//   warp 0      TMA producer: A tile 128 x 64 and B tile BN x 64 per stage, 128-byte
//               swizzle, K-major or MN-major boxes, no multicast.
//   warp 1      allocates 2*BN TMEM columns; lane 0 issues tcgen05.mma (M=128, N=BN,
//               K=16) and commits stage releases and accumulator hand-offs.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (lane quarter = warp % 4),
//               fused element-wise work, stores to global memory.
// Two accumulators in TMEM let the epilogue of one tile overlap the main loop of
// the next.  Tiles of all groups (experts) form one list that CTAs stride over;
// ragged groups take their row (or K) counts from device memory.
//
// PAIR instances run the same roles on a pair of CTAs (a cluster of two,
// cta_group::2): 256-row tiles, each CTA loading its 128 rows of A and half of B's
// columns, the leader issuing M=256 MMAs that read both CTAs' shared memory, each CTA
// draining its own 128 accumulator rows.  Per output element the pair reads a third
// fewer operand bytes into shared memory than one CTA with a 128-row tile.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

struct TmaMaps {
  CUtensorMap a[3];
  CUtensorMap b[3];
  CUtensorMap bv;
  CUtensorMap out;    // float32 / bf16 output: 32 rows x 128 bytes; SwiGLU outputs: 32 x 64 bytes
  CUtensorMap out2;   // SwiGLU backward: dB
  CUtensorMap aux_a;  // SwiGLU: saved gate pre-activation (store); backward: a (load)
  CUtensorMap aux_b;  // SwiGLU: saved value pre-activation (store); backward: b (load)
};

struct KParams {
  int M, N, groups, ragged;
  const int32_t* group_rows;
  const int32_t* group_off;  // ragged rows packed by group: group g starts at row group_off[g]
  int nseg;
  int seg_kb[3];
  int m_fastest;
  void* out;
  long long ldo, out_gs;
  void* out2;
  void* save_a;
  void* save_b;
  const void* aux_a;
  const void* aux_b;
  long long aux_ld, aux_gs;
  const float* col_add;
  const float* addend;
  long long add_ld;
  int32_t* status;
  // group g of the launch is expert (g / map_p) * map_l + map_off + g % map_p (map_p = 0:
  // expert g); one wave's experts are one launch of D * P groups
  int map_p, map_l, map_off;
  int wgrad_run;  // weight-gradient kernel: column tiles per run of a pair
};

__device__ __forceinline__ int expert_of(const KParams& p, int g) {
  return p.map_p > 0 ? (g / p.map_p) * p.map_l + p.map_off + g % p.map_p : g;
}

// Pipeline stages and staging buffers per epilogue warp of the single-CTA weight-gradient
// (write-bound) instance.
constexpr int kWbStages = 4;
constexpr int kWbBufs = 1;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kThreads = 192;  // producer warp, MMA warp, four epilogue warps

// Epilogue warps of an instance: the weight-gradient instance (both operands
// MN-major) drains 128 x 256 float32 per short tile and gets two warps per TMEM
// lane quarter, each taking half of the tile's columns.
template <bool WRITE_BOUND>
struct Roles {
  static constexpr int kEpiWarps = WRITE_BOUND ? 8 : 4;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
};
constexpr int kMaxGroups = 1024;

// WRITE_BOUND: the weight-gradient instance (both operands MN-major).  Its K is the
// few rows an expert received, so a tile's main loop is short and its output (128 x
// 256 float32 = 128 KB) weighs as much as its operands: it gets a ring of two staging
// buffers per epilogue warp so stores stream without waiting.  It never runs with
// ragged rows, so it needs no tile-prefix array.
template <int BN, bool WRITE_BOUND = false, bool SWIGLU = false, bool PAIR = false>
struct Cfg {
  static constexpr int kABytes = kBM * kBK * 2;  // 16 KB
  static constexpr int kBBytes = (PAIR ? BN / 2 : BN) * kBK * 2;  // a pair CTA holds half of B
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kStages = WRITE_BOUND ? kWbStages : ((BN == 256 && !PAIR) ? 4 : 6);
  // two accumulators; a 192-column one sits at a 256-column stride (allocations are powers of 2)
  static constexpr int kAccStride = BN <= 128 ? BN : 256;
  static constexpr int kTmemCols = 2 * kAccStride;
  static constexpr int kBufs = WRITE_BOUND ? kWbBufs : 1;  // staging buffers per epilogue warp
  static constexpr int kEpiWarps = Roles<WRITE_BOUND>::kEpiWarps;
  // a buffer holds 32 rows x 128 bytes (float32 / bf16 outputs); the forward SwiGLU
  // stages three 32 x 64-byte tiles (H, a, b), its backward three slots of two 32 x
  // 32-byte tiles (a and b in, dA and dB out in place)
  static constexpr int kBufBytes = SWIGLU ? 6144 : 4096;
  static constexpr int kStaging = kEpiWarps * kBufs * kBufBytes;
  static constexpr int kBarBytes = 8 * (2 * kStages + 5 + 12) + 16;
  static constexpr int kPrefixInts = WRITE_BOUND ? 0 : kMaxGroups + 1;
  static constexpr int kSmem = 1024 + kStages * kStage + kStaging + kBarBytes + 4 * kPrefixInts;
  static_assert(kSmem <= 232448, "shared memory budget");
};

__device__ __forceinline__ void record_status(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

struct Tile {
  int g, m, n, kb;
  int off;  // first row of group g in packed activation tensors (0 when not packed)
};

// Tile bookkeeping shared by the three roles; all of them walk the same list.
template <int BN, int EPI, int TM = kBM>
struct Sched {
  const KParams& p;
  const int* prefix;  // ragged == 1: tiles before group g (shared memory)
  int nt, mt_fixed, tiles_per_group, total;

  __device__ Sched(const KParams& pp, const int* pre) : p(pp), prefix(pre) {
    const int out_cols = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
    nt = (p.N + out_cols - 1) / out_cols;
    mt_fixed = (p.M + TM - 1) / TM;
    tiles_per_group = mt_fixed * nt;
    total = (p.ragged == 1) ? prefix[p.groups] : p.groups * tiles_per_group;
  }

  __device__ void decode(int t, int& g, int& m_tile, int& n_tile) const {
    int base, mt;
    if (p.ragged == 1) {
      int lo = 0, hi = p.groups;  // largest g with prefix[g] <= t
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= t) lo = mid; else hi = mid;
      }
      g = lo;
      base = prefix[g];
      mt = (prefix[g + 1] - prefix[g]) / nt;
    } else {
      g = t / tiles_per_group;
      base = g * tiles_per_group;
      mt = mt_fixed;
    }
    const int local = t - base;
    if (p.m_fastest) {
      m_tile = local % mt;
      n_tile = local / mt;
    } else {
      n_tile = local % nt;
      m_tile = local / nt;
    }
  }

  // everything a role needs about tile t (g = -1 past the end)
  __device__ Tile tile(int t) const {
    Tile r;
    if (t >= total) {
      r.g = -1;
      r.m = r.n = r.kb = r.off = 0;
      return r;
    }
    decode(t, r.g, r.m, r.n);
    r.g = expert_of(p, r.g);  // from here on the group is the expert
    r.kb = k_blocks(r.g);
    r.off = p.group_off != nullptr ? p.group_off[r.g] : 0;
    return r;
  }

  __device__ int k_blocks(int g) const {
    if (p.ragged == 2) {
      int r = p.group_rows[g];
      r = r < 0 ? 0 : r;
      return (r + kBK - 1) / kBK;
    }
    return p.seg_kb[0] + p.seg_kb[1] + p.seg_kb[2];
  }
};

template <int BN, bool A_MN, bool B_MN, int EPI, bool PAIR>
__global__ void __launch_bounds__(Roles<A_MN && B_MN>::kThreads, 1)
    gemm_kernel(const __grid_constant__ TmaMaps maps, const KParams p) {
  using C = Cfg<BN, A_MN && B_MN, EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_BWD, PAIR>;
  constexpr int TM = PAIR ? 2 * kBM : kBM;  // rows of A per tile (per pair of CTAs for PAIR)
  // PAIR: this CTA's rank in its cluster of two; rank 0 (the leader) issues the MMAs
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + C::kStages * C::kStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + C::kStaging);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* ebar = drain + 1;  // three per epilogue warp: its own TMA loads (SwiGLU backward)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ebar + 12);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* prefix = reinterpret_cast<int*>(staging + C::kStaging + C::kBarBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 32 * C::kEpiWarps * (PAIR ? 2 : 1));  // PAIR: both CTAs' epilogues
    }
    mbar_init(drain, 1);
    for (int w = 0; w < 12; ++w) mbar_init(&ebar[w], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < p.nseg; ++s) {
      tma_prefetch_desc(&maps.a[s]);
      tma_prefetch_desc(&maps.b[s]);
    }
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(tmem_slot, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::kTmemCols);
      tmem_relinquish();
    }
  }
  // tiles per group and their prefix (ragged rows only)
  if (C::kPrefixInts > 0 && p.ragged == 1) {
    const int out_cols = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
    const int nt = (p.N + out_cols - 1) / out_cols;
    const int per = (p.groups + kThreads - 1) / kThreads;
    const int g0 = threadIdx.x * per;
    int local = 0;
    for (int i = 0; i < per; ++i) {
      const int g = g0 + i;
      if (g < p.groups) {
        int r = p.group_rows[expert_of(p, g)];
        r = r < 0 ? 0 : (r > p.M ? p.M : r);
        local += ((r + TM - 1) / TM) * nt;
      }
    }
    // block exclusive scan of `local` over 192 threads
    __shared__ int warp_sums[kThreads / 32];
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += warp_sums[w];
    int run = before + incl - local;
    for (int i = 0; i < per; ++i) {
      const int g = g0 + i;
      if (g < p.groups) {
        prefix[g] = run;
        int r = p.group_rows[expert_of(p, g)];
        r = r < 0 ? 0 : (r > p.M ? p.M : r);
        run += ((r + TM - 1) / TM) * nt;
      }
    }
    if (threadIdx.x == kThreads - 1) prefix[p.groups] = before + incl;
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync_all();  // both CTAs' barriers exist before either touches the other's
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const volatile int* abort_v = abort_flag;

  Sched<BN, EPI, TM> sc(p, prefix);
  // both CTAs of a pair walk the same tiles: tile slots are per CTA, or per pair for PAIR
  const int slot0 = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int nslots = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int armed_phase[C::kStages];
      for (int s = 0; s < C::kStages; ++s) armed_phase[s] = -1;
      bool ok = true;
      Tile nxt = sc.tile(slot0);
      for (int t = slot0; ok && t < sc.total; t += nslots) {
        const Tile cur = nxt;
        nxt = sc.tile(t + nslots);  // issued a tile ahead: its count load overlaps this tile
        const int g = cur.g, mt = cur.m, ntile = cur.n, kb_total = cur.kb;
        // packed activations: 2-D tensors, rows offset by the group's first row
        const int gz = p.group_off != nullptr ? 0 : g, gro = cur.off;
        (void)gz;
        (void)gro;
        for (int kb = 0; kb < kb_total; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_v)) {
            ok = false;
            break;
          }
          int s = 0, kl = kb;
          if (p.ragged != 2) {
            while (s < p.nseg - 1 && kl >= p.seg_kb[s]) {
              kl -= p.seg_kb[s];
              ++s;
            }
          }
          const int k0 = kl * kBK;
          uint8_t* sa = smem + stage * C::kStage;
          uint8_t* sb = sa + C::kABytes;
          // PAIR: the leader's barrier counts both CTAs' bytes
          if (!PAIR) mbar_arrive_expect_tx(&full[stage], C::kStage);
          else if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::kStage);
          armed_phase[stage] = static_cast<int>(phase);
          const uint32_t lbar = leader_addr(smem_u32(&full[stage]));
          auto ld = [&](const CUtensorMap* map, void* dst, int c0, int c1, int c2) {
            if (PAIR) tma_load_3d_pair(map, dst, lbar, c0, c1, c2);
            else tma_load_3d(map, dst, &full[stage], c0, c1, c2);
          };
          const int m0 = mt * TM + (PAIR ? kBM * static_cast<int>(rank) : 0);
          if (!A_MN) {
            ld(&maps.a[s], sa, k0, gro + m0, gz);
          } else {
            ld(&maps.a[s], sa, m0, k0, g);
            ld(&maps.a[s], sa + 8192, m0 + 64, k0, g);
          }
          if (EPI == EPI_SWIGLU) {
            // B = [gate rows | value rows]; PAIR: the leader holds the gate half, its partner the value half
            const int n0 = ntile * (BN / 2);
            if (PAIR) {
              ld(rank == 0 ? &maps.b[0] : &maps.bv, sb, k0, n0, g);
            } else {
              ld(&maps.b[0], sb, k0, n0, g);
              ld(&maps.bv, sb + (BN / 2) * 128, k0, n0, g);
            }
          } else if (!B_MN) {
            ld(&maps.b[s], sb, k0, ntile * BN + (PAIR ? (BN / 2) * static_cast<int>(rank) : 0), g);
          } else {
            constexpr int nb = (PAIR ? BN / 2 : BN) / 64;
            const int nc0 = ntile * BN + (PAIR ? (BN / 2) * static_cast<int>(rank) : 0);
#pragma unroll
            for (int j = 0; j < nb; ++j) ld(&maps.b[s], sb + j * 8192, nc0 + 64 * j, k0, g);
          }
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(p.status, MOE_ERR_TIMEOUT);
        // let every load already issued land before the CTA goes away (PAIR: the leader's
        // barriers count both CTAs' loads, and neither CTA leaves before the other)
        if (leader)
          for (int s = 0; s < C::kStages; ++s)
            if (armed_phase[s] >= 0) mbar_wait(&full[s], static_cast<uint32_t>(armed_phase[s]), nullptr, 50000000ull);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = idesc_bf16_f32(TM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued = false;
      Tile nxt = sc.tile(slot0);
      for (int t = slot0; ok && t < sc.total; t += nslots) {
        const Tile cur = nxt;
        nxt = sc.tile(t + nslots);
        const int kb_total = cur.kb;
        if (kb_total == 0) continue;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_v)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::kAccStride);
        for (int kb = 0; kb < kb_total; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_v)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * C::kStage);
          const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t ad = A_MN ? smem_desc_sw128(a_addr + k * 2048, 8192, 1024)
                                     : smem_desc_sw128(a_addr + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc_sw128(b_addr + k * 2048, 8192, 1024)
                                     : smem_desc_sw128(b_addr + k * 32, 16, 1024);
            if (PAIR) mma_bf16_ss_pair(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
            else mma_bf16_ss(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          issued = true;
          if (PAIR) mma_commit_pair(&empty[stage]);
          else mma_commit(&empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (PAIR) mma_commit_pair(&tfull[acc]);
        else mma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(p.status, MOE_ERR_TIMEOUT);
        if (issued) {
          if (PAIR) mma_commit_pair(drain);
          else mma_commit(drain);
          mbar_wait(drain, 0, nullptr, 50000000ull);
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_in_tile = q * 32 + lane;
    const int ew = warp - 2;  // epilogue warp index
    // with eight epilogue warps, warps 2..5 take columns [0, BN/2), warps 6..9 the rest
    const int col_lo = (C::kEpiWarps == 8) ? (ew >> 2) * (BN / 2) : 0;
    const int col_hi = (C::kEpiWarps == 8) ? col_lo + BN / 2 : BN;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    // hand an accumulator back to the MMA warp (PAIR: to the leader's barrier)
    uint32_t tempty_leader = 0;
    if (PAIR)
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(tempty_leader) : "r"(smem_u32(&tempty[0])), "r"(0));
    auto release = [&](int a) {
      if (PAIR) mbar_arrive_cluster(tempty_leader + static_cast<uint32_t>(a * 8));
      else mbar_arrive(&tempty[a]);
    };
    int acc = 0;
    uint32_t acc_phase = 0;
    int ring = 0;        // next staging buffer of this warp
    uint32_t eph = 0;    // SwiGLU backward: parity of each of this warp's three load barriers
    int eslot = 0;       // SwiGLU backward: slot of the next live chunk
    Tile nxt = sc.tile(slot0);
    for (int t = slot0; t < sc.total; t += nslots) {
      const Tile cur = nxt;
      nxt = sc.tile(t + nslots);
      const int g = cur.g, mt = cur.m, ntile = cur.n, kb_total = cur.kb;
        // packed activations: 2-D tensors, rows offset by the group's first row
        const int gz = p.group_off != nullptr ? 0 : g, gro = cur.off;
        (void)gz;
        (void)gro;
      const int mbase = mt * TM + (PAIR ? kBM * static_cast<int>(rank) : 0);  // this CTA's first row
      const int row = mbase + row_in_tile;
      const bool row_ok = row < p.M;
      if (kb_total == 0) {
        // an empty contraction (group with no rows): the product is zero
        if (row_ok && (EPI == EPI_BF16 || EPI == EPI_F32)) {
          for (int c = col_lo; c < col_hi; c += 8) {
            const int col = ntile * BN + c;
            if (col >= p.N) break;
            if (EPI == EPI_BF16) {
              uint16_t* o = static_cast<uint16_t*>(p.out) + g * p.out_gs + (long long)row * p.ldo + col;
              *reinterpret_cast<uint4*>(o) = make_uint4(0, 0, 0, 0);
            } else {
              float* o = static_cast<float*>(p.out) + g * p.out_gs + (long long)row * p.ldo + col;
              reinterpret_cast<uint4*>(o)[0] = make_uint4(0, 0, 0, 0);
              reinterpret_cast<uint4*>(o)[1] = make_uint4(0, 0, 0, 0);
            }
          }
        }
        continue;
      }
      // SwiGLU backward: a and b come in by TMA one 16-column chunk ahead of their use,
      // into a ring of three slots per warp; the first chunk's load starts before the
      // accumulator is ready
      const int srow0 = mbase + q * 32;
      int s_live = 0;  // live 16-column chunks of this warp in this tile
      if constexpr (EPI == EPI_SWIGLU_BWD) {
        if (srow0 < p.M) {
          const int left = p.N - ntile * BN;
          s_live = left >= BN ? BN / 16 : (left + 15) / 16;
        }
      }
      auto swb_issue = [&](int ch, int slot) {  // lane 0
        uint8_t* sb = staging + (warp - 2) * C::kBufBytes + slot * 2048;
        uint64_t* bar = &ebar[3 * (warp - 2) + slot];
        bulk_wait_read<1>();  // the stores of the slot's previous chunk have read it
        mbar_arrive_expect_tx(bar, 2048);
        tma_load_3d(&maps.aux_a, sb, bar, ntile * BN + ch * 16, gro + srow0, gz);
        tma_load_3d(&maps.aux_b, sb + 1024, bar, ntile * BN + ch * 16, gro + srow0, gz);
      };
      if constexpr (EPI == EPI_SWIGLU_BWD) {
        if (lane == 0 && s_live > 0) swb_issue(0, eslot);
      }
      // bf16 + float32 addend: the addend of this thread's row, 64 columns at a time, is
      // loaded one piece ahead of its use; the first piece's load overlaps the MMAs
      float4 ad[EPI == EPI_BF16_ADD_F32 ? 16 : 1];
      auto load_addend = [&](int c) {
        const int col = ntile * BN + c;
        if (row_ok && col < p.N) {
          const float* src = p.addend + static_cast<long long>(row) * p.add_ld + col;
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (col + 4 * i < p.N) ad[i] = *reinterpret_cast<const float4*>(src + 4 * i);
        }
      };
      if constexpr (EPI == EPI_BF16_ADD_F32) load_addend(0);
      const bool got = mbar_wait(&tfull[acc], acc_phase, abort_v);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got)) {
        *abort_flag = 1;
        record_status(p.status, MOE_ERR_TIMEOUT);
        if constexpr (EPI == EPI_SWIGLU_BWD) {
          if (lane == 0 && s_live > 0) mbar_wait(&ebar[3 * (warp - 2) + eslot], (eph >> eslot) & 1u, nullptr, 50000000ull);
        }
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_off + static_cast<uint32_t>(acc * C::kAccStride);
      bool released = false;  // accumulator handed back to the MMA warp early

      if constexpr (EPI == EPI_SWIGLU) {
        // per chunk of 32 output columns: H, a, b as three 32 x 64-byte tiles (64-byte
        // swizzle: 16-byte piece j of row r at j ^ ((r >> 1) & 3)), three TMA stores
        const int n_out0 = ntile * (BN / 2);
        const int row0 = mbase + q * 32;
        uint8_t* buf = staging + ew * C::kBufBytes;
        const uint32_t rbase = smem_u32(buf) + lane * 64;
        const int sw = (lane >> 1) & 3;
#pragma unroll 1
        for (int c2 = 0; c2 < BN / 2; c2 += 64) {
          // two chunks of gate and value columns (four TMEM loads) per wait
          uint32_t rg[2][32], ru[2][32];
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            tmem_ld_32cols_async(tbase + c2 + 32 * i, rg[i]);
            tmem_ld_32cols_async(tbase + BN / 2 + c2 + 32 * i, ru[i]);
          }
          tmem_wait_ld();
          if (c2 + 64 >= BN / 2) {
            tc_fence_before();
            release(acc);
            released = true;
          }
#pragma unroll
          for (int i = 0; i < 2; ++i) {
          const int c = c2 + 32 * i;
          uint32_t h[16], ga[16], gb[16];
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            const float a0 = __uint_as_float(rg[i][2 * e2]), a1 = __uint_as_float(rg[i][2 * e2 + 1]);
            const float u0 = __uint_as_float(ru[i][2 * e2]), u1 = __uint_as_float(ru[i][2 * e2 + 1]);
            const float s0 = __fdividef(a0, 1.0f + __expf(-a0)), s1 = __fdividef(a1, 1.0f + __expf(-a1));
            h[e2] = pack_bf16x2(s0 * u0, s1 * u1);
            ga[e2] = pack_bf16x2(a0, a1);
            gb[e2] = pack_bf16x2(u0, u1);
          }
          if (lane == 0) bulk_wait_read<0>();  // the previous chunk's stores have read the buffer
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t off = ((j ^ sw) << 4);
            st_shared_v4(rbase + off, h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
            st_shared_v4(rbase + 2048 + off, ga[4 * j], ga[4 * j + 1], ga[4 * j + 2], ga[4 * j + 3]);
            st_shared_v4(rbase + 4096 + off, gb[4 * j], gb[4 * j + 1], gb[4 * j + 2], gb[4 * j + 3]);
          }
          fence_async_shared();
          __syncwarp();
          const int col0 = n_out0 + c;
          if (lane == 0 && col0 < p.N && row0 < p.M) {
            tma_store_3d(&maps.out, buf, col0, gro + row0, gz);
            if (p.save_a != nullptr) {
              tma_store_3d(&maps.aux_a, buf + 2048, col0, gro + row0, gz);
              tma_store_3d(&maps.aux_b, buf + 4096, col0, gro + row0, gz);
            }
            bulk_commit();
          }
          }
        }
      } else if constexpr ((EPI == EPI_F32 || EPI == EPI_BF16) && (A_MN && B_MN)) {
        // Weight gradients: each tile's short main loop is worth less than its 128 KB
        // result, and TMA stores would queue the next tile's operand loads behind them.
        // The result leaves through the load/store path instead: one 32-column chunk at
        // a time, staged as 32 rows x 128 bytes (128-byte swizzle: 16-byte piece j of
        // row r at j ^ (r & 7)) and read back four rows per instruction, so every store
        // instruction writes four whole 128-byte lines.
        constexpr int kChunk = (EPI == EPI_F32) ? 32 : 64;
        constexpr int kEsz = (EPI == EPI_F32) ? 4 : 2;
        const int row0 = mbase + q * 32;
        uint8_t* buf = staging + ew * C::kBufs * C::kBufBytes;
        const uint32_t sbase = smem_u32(buf);
        const int piece = lane & 7;    // 16-byte piece of a row this lane reads back
        const int rsub = lane >> 3;    // row within each group of four
        char* obase = static_cast<char*>(p.out) + static_cast<long long>(g) * p.out_gs * kEsz;
#pragma unroll 1
        for (int c = col_lo; c < col_hi; c += kChunk) {
          const int col0 = ntile * BN + c;
          if (col0 >= p.N || row0 >= p.M) break;
          uint32_t w[32];
          __syncwarp();
          if constexpr (EPI == EPI_F32) {
            float v[32];
            tmem_ld_32cols(tbase + c, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(v[i]);
          } else {
            float v0[32], v1[32];
            tmem_ld_32cols(tbase + c, v0);
            tmem_ld_32cols(tbase + c + 32, v1);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              w[i] = pack_bf16x2(v0[2 * i], v0[2 * i + 1]);
              w[16 + i] = pack_bf16x2(v1[2 * i], v1[2 * i + 1]);
            }
          }
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(sbase + lane * 128 + ((j ^ (lane & 7)) << 4), w[4 * j], w[4 * j + 1], w[4 * j + 2],
                         w[4 * j + 3]);
          __syncwarp();
          const int col = col0 + piece * (16 / kEsz);
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int r = it * 4 + rsub;
            uint32_t a0, a1, a2, a3;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                         : "r"(sbase + r * 128 + ((piece ^ (r & 7)) << 4)));
            const int row = row0 + r;
            if (row < p.M && col < p.N)
              *reinterpret_cast<uint4*>(obase + (static_cast<long long>(row) * p.ldo + col) * kEsz) =
                  make_uint4(a0, a1, a2, a3);
          }
        }
      } else if constexpr (EPI == EPI_F32 || EPI == EPI_BF16 || EPI == EPI_BF16_ADD_F32) {
        // Four TMEM loads (128 columns) in flight before one wait, then the 128 columns
        // leave through shared memory: 32 rows x 128 bytes per staging buffer (128-byte
        // swizzle: 16-byte piece j of row r at j ^ (r & 7)), one TMA tensor store each.
        // Rows past M and columns past N are clipped by the tensor map.  The accumulator
        // is released as soon as the whole tile is in registers.  With an addend, each
        // 64-column piece gets its float32 addend before rounding to bf16.
        constexpr int kChunk = (EPI == EPI_F32) ? 32 : 64;  // columns per 128-byte row
        // columns per TMEM wait (the addend's registers leave room for 64; a 192-column tile
        // drains in three spans)
        constexpr int kSpan = (EPI == EPI_BF16_ADD_F32 || BN % 128 != 0) ? 64 : 128;
        const int row0 = mbase + q * 32;
#pragma unroll 1
        for (int half = 0; half < BN; half += kSpan) {
          uint32_t r[kSpan / 32][32];
          __syncwarp();
#pragma unroll
          for (int i = 0; i < kSpan / 32; ++i) tmem_ld_32cols_async(tbase + half + 32 * i, r[i]);
          tmem_wait_ld();
          if (half + kSpan >= BN) {
            tc_fence_before();
            release(acc);
            released = true;
          }
#pragma unroll
          for (int cc = 0; cc < kSpan / kChunk; ++cc) {
            uint32_t w[32];
            const int col0 = ntile * BN + half + cc * kChunk;
            // see the weight-gradient path: no buffer write without a committed store
            if (col0 >= p.N || row0 >= p.M) continue;
            if constexpr (EPI == EPI_F32) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                float x = __uint_as_float(r[cc][i]);
                if (p.col_add != nullptr && col0 + i < p.N) x += p.col_add[col0 + i];
                w[i] = __float_as_uint(x);
              }
            } else {
              if constexpr (EPI == EPI_BF16_ADD_F32) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  uint32_t* x = &r[2 * cc + (i >> 3)][4 * (i & 7)];
                  x[0] = __float_as_uint(__uint_as_float(x[0]) + ad[i].x);
                  x[1] = __float_as_uint(__uint_as_float(x[1]) + ad[i].y);
                  x[2] = __float_as_uint(__uint_as_float(x[2]) + ad[i].z);
                  x[3] = __float_as_uint(__uint_as_float(x[3]) + ad[i].w);
                }
                if (half + (cc + 1) * kChunk < BN) load_addend(half + (cc + 1) * kChunk);
              }
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                w[i] = pack_bf16x2(__uint_as_float(r[2 * cc][2 * i]), __uint_as_float(r[2 * cc][2 * i + 1]));
                w[16 + i] =
                    pack_bf16x2(__uint_as_float(r[2 * cc + 1][2 * i]), __uint_as_float(r[2 * cc + 1][2 * i + 1]));
              }
            }
            uint8_t* buf = staging + (ew * C::kBufs + ring) * C::kBufBytes;
            if (++ring == C::kBufs) ring = 0;
            const uint32_t row_addr = smem_u32(buf) + lane * 128;
            // the store that last used this buffer (kBufs chunks ago) has read it
            if (lane == 0) bulk_wait_read<C::kBufs - 1>();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              st_shared_v4(row_addr + ((j ^ (lane & 7)) << 4), w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
            fence_async_shared();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&maps.out, buf, col0, gro + row0, gz);
              bulk_commit();
            }
          }
        }
      } else if constexpr (EPI == EPI_SWIGLU_BWD) {
        // per chunk of 16 columns: dH from TMEM, a and b from the slot loaded one chunk
        // ago (32 x 32-byte tiles, unswizzled), dA and dB formed in place and TMA-stored
        const int wi = warp - 2;
        bool ok = true;
#pragma unroll 1
        for (int ch = 0; ch < s_live; ++ch) {  // the live chunks are a prefix (warp-uniform)
          uint32_t r[16];
          __syncwarp();
          tmem_ld_16cols(tbase + ch * 16, r);
          const int slot = eslot;
          eslot = eslot == 2 ? 0 : eslot + 1;
          if (lane == 0 && ch + 1 < s_live) swb_issue(ch + 1, eslot);
          const bool gotc = mbar_wait(&ebar[3 * wi + slot], (eph >> slot) & 1u, abort_v);
          eph ^= 1u << slot;
          if (!__all_sync(0xffffffffu, gotc)) {
            // let the next chunk's load land before leaving
            if (lane == 0 && ch + 1 < s_live) mbar_wait(&ebar[3 * wi + eslot], (eph >> eslot) & 1u, nullptr, 50000000ull);
            ok = false;
            break;
          }
          uint8_t* sb = staging + wi * C::kBufBytes + slot * 2048;
          const uint32_t ra = smem_u32(sb) + lane * 32;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            uint32_t aw[4], bw[4], da[4], db[4];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(aw[0]), "=r"(aw[1]), "=r"(aw[2]), "=r"(aw[3]) : "r"(ra + 16 * j));
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(bw[0]), "=r"(bw[1]), "=r"(bw[2]), "=r"(bw[3]) : "r"(ra + 1024 + 16 * j));
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              float rda[2], rdb[2];
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                const float a = hh ? bf16_hi(aw[w]) : bf16_lo(aw[w]);
                const float b = hh ? bf16_hi(bw[w]) : bf16_lo(bw[w]);
                const float dh = __uint_as_float(r[8 * j + 2 * w + hh]);
                const float sg = __fdividef(1.0f, 1.0f + __expf(-a));
                rda[hh] = dh * b * (sg * (1.0f + a * (1.0f - sg)));
                rdb[hh] = dh * (a * sg);
              }
              da[w] = pack_bf16x2(rda[0], rda[1]);
              db[w] = pack_bf16x2(rdb[0], rdb[1]);
            }
            st_shared_v4(ra + 16 * j, da[0], da[1], da[2], da[3]);
            st_shared_v4(ra + 1024 + 16 * j, db[0], db[1], db[2], db[3]);
          }
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&maps.out, sb, ntile * BN + ch * 16, gro + srow0, gz);
            tma_store_3d(&maps.out2, sb + 1024, ntile * BN + ch * 16, gro + srow0, gz);
            bulk_commit();
          }
        }
        if (!ok) {
          *abort_flag = 1;
          record_status(p.status, MOE_ERR_TIMEOUT);
          break;
        }
      } else {
        static_assert(EPI < 0, "an epilogue without a branch");
      }
      __syncwarp();
      if (!released) {
        tc_fence_before();
        release(acc);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_all();  // every store of this warp has completed
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync_all();  // neither CTA leaves while the other may still touch its memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else tmem_dealloc(tmem_base, C::kTmemCols);
  }
}


// ====================================================================== weight gradients on CTA pairs
//
// dW = A^T B with both operands MN-major and a float32 result, on a pair of CTAs (one
// cluster of two, cta_group::2): 256 x 256 output tiles, each CTA loading 128 rows of A
// and 128 of B's 256 columns per k-block, the leader issuing M=256 tcgen05.mma that read
// both CTAs' shared memory, each CTA draining its 128 accumulator rows.  Per output
// element this reads a third fewer operand bytes than the single-CTA kernel, which is
// what bounds these short (rows-per-expert) contractions.
constexpr int kPairEpiWarps = 8;
constexpr int kPairThreads = 64 + 32 * kPairEpiWarps;

struct PairCfg {
  static constexpr int kABytes = 128 * kBK * 2;
  static constexpr int kBBytes = 128 * kBK * 2;
  static constexpr int kStage = kABytes + kBBytes;  // 32 KB per CTA
  static constexpr int kStages = 6;
  static constexpr int kTmemCols = 512;             // two 256-column accumulators
  static constexpr int kStaging = kPairEpiWarps * 4096;
  static constexpr int kBarBytes = 8 * (2 * kStages + 5) + 16;
  static constexpr int kSmem = 1024 + kStages * kStage + kStaging + kBarBytes;
  static_assert(kSmem <= 232448, "shared memory budget");
};

// An epilogue warp's share of a pair tile: 32 rows (row0..) x 128 columns (col_lo..) of
// this CTA's accumulator half, per 32-column chunk TMEM -> registers -> staging -> one
// TMA store (the copy engine clips rows and columns past the output's edge).
__device__ __forceinline__ void pair_drain(const TmaMaps& maps, const KParams& p, uint32_t tbase, int col_lo,
                                           int ntile, int row0, int g, uint8_t* buf, uint32_t row_addr, int lane) {
#pragma unroll 1
  for (int c = col_lo; c < col_lo + 128; c += 32) {
    const int col0 = ntile * 256 + c;
    if (col0 >= p.N || row0 >= p.M) break;
    float v[32];
    if (lane == 0) bulk_wait_read<0>();  // the previous chunk's store has read the buffer
    __syncwarp();
    tmem_ld_32cols(tbase + c, v);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      st_shared_v4(row_addr + ((j ^ (lane & 7)) << 4), __float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]),
                   __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3]));
    fence_async_shared();
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(&maps.out, buf, col0, row0, g);
      bulk_commit();
    }
  }
}

// the same share of a tile whose contraction is empty: zeros
__device__ __forceinline__ void pair_zero(const KParams& p, int col_lo, int ntile, int row0, int g, int lane) {
  float* obase = static_cast<float*>(p.out) + static_cast<long long>(g) * p.out_gs;
  const int row = row0 + lane;
  if (row < p.M)
    for (int c = col_lo; c < col_lo + 128; c += 4) {
      const int col = ntile * 256 + c;
      if (col >= p.N) break;
      *reinterpret_cast<float4*>(obase + static_cast<long long>(row) * p.ldo + col) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// Tiles of a pair come in runs: up to p.wgrad_run consecutive column tiles of one row
// tile of one group.  When a group's whole contraction fits the stage ring (k-blocks <=
// kStages), the run's first tile loads A and B into stages 0..kb-1 and its other tiles
// load only B: the A panel (this CTA's 128 rows x K) stays in shared memory for the run.
// Runs of two measured 4% faster than single tiles on the routed weight gradients (K =
// an expert's rows); longer runs leave pairs idle, and the dense weight gradients (K = T)
// take single tiles.

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    gemm_pair_wgrad_kernel(const __grid_constant__ TmaMaps maps, const KParams p) {
  using C = PairCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + C::kStages * C::kStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + C::kStaging);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 32 * kPairEpiWarps);  // both CTAs' epilogue threads
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.a[0]);
    tma_prefetch_desc(&maps.b[0]);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before either touches the other's
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const volatile int* abort_v = abort_flag;

  const int mt_n = (p.M + 255) / 256;
  const int nt_n = (p.N + 255) / 256;
  const int run_len = p.wgrad_run > 1 ? p.wgrad_run : 1;
  const int nrun = (nt_n + run_len - 1) / run_len;  // runs per row tile
  const int runs = p.groups * mt_n * nrun;
  auto k_blocks = [&](int g) {
    if (p.ragged == 2) {
      const int r = p.group_rows[g];
      return r > 0 ? (r + kBK - 1) / kBK : 0;
    }
    return p.seg_kb[0];
  };
  // Runs are ordered column-run fastest, so the pairs working at one time cover whole
  // rows of the result.  Every role fetches a run one step ahead, so the load of a
  // group's row count overlaps the run before it.
  struct PairRun {
    int g, m, n0, n1, kb;
    int off;       // first K row of group g in packed activation tensors (0 when not packed)
    bool resident;  // the A panel stays in stages 0..kb-1 for the whole run
  };
  auto fetch = [&](int u) {
    PairRun r{0, 0, 0, 0, 0, 0, false};
    if (u < runs) {
      const int per_group = mt_n * nrun;
      int g = u / per_group;
      const int l = u - g * per_group;
      r.m = l / nrun;
      r.n0 = (l % nrun) * run_len;
      r.n1 = min(nt_n, r.n0 + run_len);
      g = expert_of(p, g);
      r.g = g;
      r.kb = k_blocks(g);
      r.off = p.group_off != nullptr ? p.group_off[g] : 0;
      r.resident = r.n1 - r.n0 > 1 && r.kb <= C::kStages;
    }
    return r;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;          // next ring stage (runs that do not keep A)
      uint32_t use_bits = 0;  // per stage: parity of its fills so far
      int armed_phase[C::kStages];
      for (int s = 0; s < C::kStages; ++s) armed_phase[s] = -1;
      bool ok = true;
      PairRun nxt = fetch(pair);
      for (int u = pair; ok && u < runs; u += npairs) {
        const PairRun cur = nxt;
        nxt = fetch(u + npairs);
        const int g = cur.g, kb_total = cur.kb;
        // packed activations: 2-D tensors, rows offset by the group's first row
        const int gz = p.group_off != nullptr ? 0 : g, gro = cur.off;
        const int m0 = cur.m * 256 + 128 * static_cast<int>(rank);
        for (int nt = cur.n0; ok && nt < cur.n1; ++nt) {
          const bool load_a = !cur.resident || nt == cur.n0;
          const int n0 = nt * 256 + 128 * static_cast<int>(rank);
          if (cur.resident) stage = 0;
          for (int kb = 0; kb < kb_total; ++kb) {
            const uint32_t par = (use_bits >> stage) & 1u;
            if (!mbar_wait(&empty[stage], par ^ 1u, abort_v)) {
              ok = false;
              break;
            }
            use_bits ^= 1u << stage;
            const uint32_t bytes = load_a ? 2 * C::kStage : 2 * C::kBBytes;
            if (leader) mbar_arrive_expect_tx(&full[stage], bytes);
            armed_phase[stage] = static_cast<int>(par);
            const uint32_t bar = leader_addr(smem_u32(&full[stage]));
            uint8_t* sa = smem + stage * C::kStage;
            uint8_t* sb = sa + C::kABytes;
            const int k0 = kb * kBK;
            if (load_a) {
              tma_load_3d_pair(&maps.a[0], sa, bar, m0, gro + k0, gz);
              tma_load_3d_pair(&maps.a[0], sa + 8192, bar, m0 + 64, gro + k0, gz);
            }
            tma_load_3d_pair(&maps.b[0], sb, bar, n0, gro + k0, gz);
            tma_load_3d_pair(&maps.b[0], sb + 8192, bar, n0 + 64, gro + k0, gz);
            if (++stage == C::kStages) stage = 0;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(p.status, MOE_ERR_TIMEOUT);
        // the leader's full barriers count both CTAs' bytes: let every armed load land
        if (leader)
          for (int s = 0; s < C::kStages; ++s)
            if (armed_phase[s] >= 0)
              mbar_wait(&full[s], static_cast<uint32_t>(armed_phase[s]), nullptr, 50000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, 256, true, true);
      int stage = 0;
      uint32_t use_bits = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued = false;
      PairRun nxt = fetch(pair);
      for (int u = pair; ok && u < runs; u += npairs) {
        const PairRun cur = nxt;
        nxt = fetch(u + npairs);
        const int kb_total = cur.kb;
        if (kb_total == 0) continue;
        for (int nt = cur.n0; ok && nt < cur.n1; ++nt) {
          if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_v)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
          if (cur.resident) stage = 0;
          for (int kb = 0; kb < kb_total; ++kb) {
            if (!mbar_wait(&full[stage], (use_bits >> stage) & 1u, abort_v)) {
              ok = false;
              break;
            }
            use_bits ^= 1u << stage;
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + stage * C::kStage);
            const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              const uint64_t ad = smem_desc_sw128(a_addr + k * 2048, 8192, 1024);
              const uint64_t bd = smem_desc_sw128(b_addr + k * 2048, 8192, 1024);
              mma_bf16_ss_pair(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
            }
            issued = true;
            mma_commit_pair(&empty[stage]);
            if (++stage == C::kStages) stage = 0;
          }
          if (!ok) break;
          mma_commit_pair(&tfull[acc]);
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1u;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(p.status, MOE_ERR_TIMEOUT);
        if (issued) {
          mma_commit_pair(drain);
          mbar_wait(drain, 0, nullptr, 50000000ull);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int ew = warp - 2;
    const int col_lo = (ew >> 2) * 128;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint8_t* buf = staging + ew * 4096;  // one 32 x 32 float32 chunk, rows swizzled as the TMA expects
    const uint32_t row_addr = smem_u32(buf) + lane * 128;
    uint32_t tempty_leader;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(tempty_leader) : "r"(smem_u32(&tempty[0])), "r"(0));
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    PairRun nxt = fetch(pair);
    for (int u = pair; ok && u < runs; u += npairs) {
      const PairRun cur = nxt;
      nxt = fetch(u + npairs);
      const int g = cur.g;
      const int row0 = cur.m * 256 + 128 * static_cast<int>(rank) + q * 32;
      for (int nt = cur.n0; nt < cur.n1; ++nt) {
        if (cur.kb == 0) {
          pair_zero(p, col_lo, nt, row0, g, lane);
          continue;
        }
        const bool got = mbar_wait(&tfull[acc], acc_phase, abort_v);
        __syncwarp();
        if (!__all_sync(0xffffffffu, got)) {
          *abort_flag = 1;
          record_status(p.status, MOE_ERR_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        pair_drain(maps, p, tmem_base + lane_off + static_cast<uint32_t>(acc * 256), col_lo, nt, row0, g, buf,
                   row_addr, lane);
        __syncwarp();
        tc_fence_before();
        // hand the accumulator back to the leader's MMA warp
        mbar_arrive_cluster(tempty_leader + static_cast<uint32_t>(acc * 8));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  }

  if (warp >= 2 && lane == 0) bulk_wait_all();  // every store has landed before the CTA exits
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the other may still touch its memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}


// ====================================================================== host side

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

moe_status_t make_map(CUtensorMap* m, const Mat& t, uint32_t box_inner, uint32_t box_rows, const char* what,
                      CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, int esize = 2,
                      CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  if (t.ptr == nullptr) return fail(MOE_ERR_INVALID_ARG, std::string("gemm operand is null: ") + what);
  if ((reinterpret_cast<uintptr_t>(t.ptr) & 15) != 0)
    return fail(MOE_ERR_INVALID_ARG, std::string("gemm operand not 16-byte aligned: ") + what);
  if (t.inner <= 0 || t.rows <= 0 || t.groups <= 0 || t.ld < t.inner || (t.ld * esize) % 16 != 0 ||
      (t.gs * esize) % 16 != 0)
    return fail(MOE_ERR_INVALID_ARG, std::string("gemm operand has a bad shape or stride: ") + what);
  auto fn = encode_fn();
  if (fn == nullptr) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(t.inner), static_cast<cuuint64_t>(t.rows),
                        static_cast<cuuint64_t>(t.groups)};
  const int64_t gs = t.groups > 1 ? t.gs : t.ld * t.rows;
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(t.ld * esize), static_cast<cuuint64_t>(gs * esize)};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dtype, 3, const_cast<void*>(t.ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MOE_ERR_CUDA, std::string("cuTensorMapEncodeTiled failed for ") + what + " (" +
                                  std::to_string(static_cast<int>(r)) + ")");
  return MOE_OK;
}

// tiles: output tiles of the launch (pair tiles for PAIR); the grid is one CTA (or pair)
// per tile up to what fits on the device at once
template <int BN, bool A_MN, bool B_MN, int EPI, bool PAIR>
moe_status_t launch_instance(const TmaMaps& maps, const KParams& kp, long long tiles, cudaStream_t st) {
  auto kern = gemm_kernel<BN, A_MN, B_MN, EPI, PAIR>;
  const int smem = Cfg<BN, A_MN && B_MN, EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_BWD, PAIR>::kSmem;
  constexpr int threads = Roles<A_MN && B_MN>::kThreads;
  static std::atomic<uint64_t> attr_done{0};  // per instantiation, one bit per device
  const moe_status_t r = ensure_max_smem(reinterpret_cast<const void*>(kern), smem, attr_done, "gemm");
  if (r != MOE_OK) return r;
  if (!PAIR) {
    const int grid = static_cast<int>(std::min<long long>(tiles, device_sm_count()));
    kern<<<grid, threads, smem, st>>>(maps, kp);
    count_launch();
    return cuda_check(cudaGetLastError(), "gemm launch");
  }
  // pairs that fit on the device at once, per device (0: not asked yet)
  static std::atomic<int> max_pairs_dev[kMaxDevices];
  const int dev = current_device();
  int max_pairs = (dev >= 0 && dev < kMaxDevices) ? max_pairs_dev[dev].load(std::memory_order_relaxed) : 0;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (max_pairs == 0) {
    cfg.gridDim = dim3(2 * (device_sm_count() / 2));
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) != cudaSuccess || nc <= 0) {
      (void)cudaGetLastError();
      nc = device_sm_count() / 2;
    }
    max_pairs = std::min(nc, device_sm_count() / 2);
    if (dev >= 0 && dev < kMaxDevices) max_pairs_dev[dev].store(max_pairs, std::memory_order_relaxed);
  }
  const int pairs = static_cast<int>(std::min<long long>(tiles, max_pairs));
  cfg.gridDim = dim3(2 * pairs);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, maps, kp);
  count_launch();
  if (e != cudaSuccess) return cuda_check(e, "pair gemm launch");
  return cuda_check(cudaGetLastError(), "pair gemm launch");
}

}  // namespace

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return -1;
  }
  return dev;
}

moe_status_t ensure_max_smem(const void* func, int bytes, std::atomic<uint64_t>& done_mask, const char* what) {
  const int dev = current_device();
  const uint64_t bit = (dev >= 0 && dev < kMaxDevices) ? (uint64_t(1) << dev) : 0;
  if (bit != 0 && (done_mask.load(std::memory_order_acquire) & bit)) return MOE_OK;
  const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_check(e, (std::string("cudaFuncSetAttribute(") + what + ")").c_str());
  if (bit != 0) done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return MOE_OK;
}

int device_sm_count() {
  static std::atomic<int> cached[kMaxDevices];  // 0: not looked up yet
  const int dev = current_device();
  if (dev >= 0 && dev < kMaxDevices) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (dev < 0 || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = 148;
  }
  if (dev >= 0 && dev < kMaxDevices) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

moe_status_t gemm_run(const GemmArgs& a, cudaStream_t st) {
  if (a.M <= 0 || a.N <= 0 || a.groups <= 0) return MOE_OK;
  if (a.bn != 128 && a.bn != 256 &&
      !(a.bn == 192 && a.pair && !a.a_mn && !a.b_mn && a.epi == EPI_F32 && a.nseg == 1))
    return fail(MOE_ERR_UNSUPPORTED,
                "gemm tile width must be 128 or 256 (192: CTA pairs, K-major operands, float32 out)");
  if (a.groups > kMaxGroups) return fail(MOE_ERR_UNSUPPORTED, "too many gemm groups");
  if (a.nseg < 1 || a.nseg > 3) return fail(MOE_ERR_INVALID_ARG, "gemm needs 1..3 K segments");
  if (a.ragged != 0 && a.group_rows == nullptr) return fail(MOE_ERR_INVALID_ARG, "ragged gemm needs group rows");
  if (a.ragged == 2 && a.nseg != 1) return fail(MOE_ERR_INVALID_ARG, "ragged-K gemm takes one segment");
  // packed groups: activations are 2-D (rows_total rows), weights 3-D; only the epilogues
  // and kernels that address activation rows through tensor maps take them
  const bool packed = a.group_off != nullptr;
  if (packed && (a.ragged == 0 || a.rows_total <= 0 || a.epi == EPI_BF16_ADD_F32 ||
                 (a.ragged == 2 && !(a.a_mn && a.b_mn && a.epi == EPI_F32 && a.bn == 256))))
    return fail(MOE_ERR_UNSUPPORTED, "packed groups need ragged rows or a ragged-K weight gradient");
  if (a.epi == EPI_SWIGLU && (a.nseg != 1 || a.b_mn || a.N % (a.bn / 2) != 0))
    return fail(MOE_ERR_UNSUPPORTED, "SwiGLU gemm needs one K-major segment and N a multiple of BN/2");
  if (a.N % 8 != 0) return fail(MOE_ERR_UNSUPPORTED, "gemm N must be a multiple of 8");
  if (a.a_mn && a.b_mn && a.ragged == 1)
    return fail(MOE_ERR_UNSUPPORTED, "gemm with both operands MN-major takes no ragged rows");
  if (a.out == nullptr) return fail(MOE_ERR_INVALID_ARG, "gemm output is null");

  // groups of the output and element-wise tensors (a launch may cover some of them)
  const int tgroups = a.tensor_groups > 0 ? a.tensor_groups : a.groups;
  TmaMaps maps;
  memset(&maps, 0, sizeof(maps));
  KParams kp;
  memset(&kp, 0, sizeof(kp));
  kp.M = a.M;
  kp.N = a.N;
  kp.groups = a.groups;
  kp.ragged = a.ragged;
  kp.group_rows = a.group_rows;
  kp.group_off = a.group_off;
  kp.nseg = a.nseg;
  for (int s = 0; s < a.nseg; ++s) {
    moe_status_t r;
    r = make_map(&maps.a[s], a.A[s], 64, a.a_mn ? 64 : 128, "A");
    if (r != MOE_OK) return r;
    // a pair CTA loads half of B's rows (SwiGLU: the gate or the value half)
    const uint32_t b_rows = a.b_mn ? 64 : ((a.epi == EPI_SWIGLU || a.pair) ? a.bn / 2 : a.bn);
    r = make_map(&maps.b[s], a.B[s], 64, b_rows, "B");
    if (r != MOE_OK) return r;
    kp.seg_kb[s] = a.ragged == 2 ? 0 : static_cast<int>((a.K[s] + kBK - 1) / kBK);
  }
  if (a.epi == EPI_SWIGLU) {
    moe_status_t r = make_map(&maps.bv, a.Bv, 64, a.bn / 2, "B value");
    if (r != MOE_OK) return r;
  }
  if (a.epi == EPI_SWIGLU || a.epi == EPI_SWIGLU_BWD) {
    // 32 x 32 bf16 tiles (64-byte rows) of the element-wise operands and results
    auto tile = [&](CUtensorMap* m, const void* ptr, int64_t ld, int64_t gs, const char* what) {
      Mat o;
      o.ptr = ptr;
      o.inner = a.N;
      o.rows = packed ? a.rows_total : a.M;
      o.groups = packed ? 1 : tgroups;
      o.ld = ld;
      o.gs = (tgroups > 1 && !packed) ? gs : ld * o.rows;
      return make_map(m, o, 32, 32, what, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, CU_TENSOR_MAP_SWIZZLE_64B);
    };
    moe_status_t r = tile(&maps.out, a.out, a.ldo, a.out_gs, "output");
    if (r != MOE_OK) return r;
    if (a.epi == EPI_SWIGLU && a.save_a != nullptr) {
      if (a.save_b == nullptr) return fail(MOE_ERR_INVALID_ARG, "SwiGLU saves both pre-activations or neither");
      if ((r = tile(&maps.aux_a, a.save_a, a.ldo, a.out_gs, "saved gate")) != MOE_OK) return r;
      if ((r = tile(&maps.aux_b, a.save_b, a.ldo, a.out_gs, "saved value")) != MOE_OK) return r;
    }
    if (a.epi == EPI_SWIGLU_BWD) {
      // 32 rows x 16 columns (32-byte rows, unswizzled) for the chunked backward epilogue
      auto tile16 = [&](CUtensorMap* m, const void* ptr, int64_t ld, int64_t gs, const char* what) {
        Mat o;
        o.ptr = ptr;
        o.inner = a.N;
        o.rows = packed ? a.rows_total : a.M;
        o.groups = packed ? 1 : tgroups;
        o.ld = ld;
        o.gs = (tgroups > 1 && !packed) ? gs : ld * o.rows;
        return make_map(m, o, 16, 32, what, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, CU_TENSOR_MAP_SWIZZLE_NONE);
      };
      if ((r = tile16(&maps.out, a.out, a.ldo, a.out_gs, "dA")) != MOE_OK) return r;
      if ((r = tile16(&maps.out2, a.out2, a.ldo, a.out_gs, "dB")) != MOE_OK) return r;
      if ((r = tile16(&maps.aux_a, a.aux_a, a.aux_ld, a.aux_gs, "a")) != MOE_OK) return r;
      if ((r = tile16(&maps.aux_b, a.aux_b, a.aux_ld, a.aux_gs, "b")) != MOE_OK) return r;
    }
  }
  if (a.epi == EPI_F32 || a.epi == EPI_BF16 || a.epi == EPI_BF16_ADD_F32) {
    Mat o;
    o.ptr = a.out;
    o.inner = a.N;
    // a packed ragged-row output is 2-D; a weight gradient's output stays one per group
    const bool packed_out = packed && a.ragged == 1;
    o.rows = packed_out ? a.rows_total : a.M;
    o.groups = packed_out ? 1 : tgroups;
    o.ld = a.ldo;
    o.gs = (tgroups > 1 && !packed_out) ? a.out_gs : a.ldo * o.rows;
    moe_status_t r = a.epi == EPI_F32
                         ? make_map(&maps.out, o, 32, 32, "output", CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4)
                         : make_map(&maps.out, o, 64, 32, "output");
    if (r != MOE_OK) return r;
  }
  kp.m_fastest = a.m_fastest ? 1 : 0;
  kp.out = a.out;
  kp.ldo = a.ldo;
  kp.out_gs = a.out_gs;
  kp.out2 = a.out2;
  kp.save_a = a.save_a;
  kp.save_b = a.save_b;
  kp.aux_a = a.aux_a;
  kp.aux_b = a.aux_b;
  kp.aux_ld = a.aux_ld;
  kp.aux_gs = a.aux_gs;
  kp.col_add = a.col_add;
  kp.addend = a.addend;
  kp.add_ld = a.add_ld;
  kp.status = a.status;
  kp.map_p = a.map_p;
  kp.map_l = a.map_l;
  kp.map_off = a.map_off;

  if (a.a_mn && a.b_mn && a.epi == EPI_F32 && a.nseg == 1 && a.ragged != 1 && a.bn == 256) {
    // runs of up to wgrad_run column tiles: one pair each
    kp.wgrad_run = a.ragged == 2 ? 2 : 1;
    const long long pair_runs = static_cast<long long>(a.groups) * ((a.M + 255) / 256) *
                                ((((a.N + 255) / 256) + kp.wgrad_run - 1) / kp.wgrad_run);
    // pairs that fit on the device at once, per device (0: not measured yet)
    static std::atomic<int> max_pairs_dev[kMaxDevices];
    static std::atomic<uint64_t> attr_done{0};
    const int dev = current_device();
    int max_pairs = (dev >= 0 && dev < kMaxDevices) ? max_pairs_dev[dev].load(std::memory_order_relaxed) : 0;
    {
      const moe_status_t r = ensure_max_smem(reinterpret_cast<const void*>(gemm_pair_wgrad_kernel), PairCfg::kSmem,
                                             attr_done, "pair gemm");
      if (r != MOE_OK) return r;
    }
    if (max_pairs == 0) {
      cudaLaunchConfig_t cfg;
      memset(&cfg, 0, sizeof(cfg));
      cfg.gridDim = dim3(2 * (device_sm_count() / 2));
      cfg.blockDim = dim3(kPairThreads);
      cfg.dynamicSmemBytes = PairCfg::kSmem;
      int nc = 0;
      if (cudaOccupancyMaxActiveClusters(&nc, gemm_pair_wgrad_kernel, &cfg) != cudaSuccess || nc <= 0) {
        (void)cudaGetLastError();
        nc = device_sm_count() / 2;
      }
      max_pairs = std::min(nc, device_sm_count() / 2);
      if (dev >= 0 && dev < kMaxDevices) max_pairs_dev[dev].store(max_pairs, std::memory_order_relaxed);
    }
    const int pairs = static_cast<int>(std::min<long long>(pair_runs, max_pairs));
    if (pairs <= 0) return MOE_OK;
    gemm_pair_wgrad_kernel<<<2 * pairs, kPairThreads, PairCfg::kSmem, st>>>(maps, kp);
    count_launch();
    return cuda_check(cudaGetLastError(), "pair gemm launch");
  }
  const int out_cols = a.epi == EPI_SWIGLU ? a.bn / 2 : a.bn;
  const int tm = a.pair ? 2 * kBM : kBM;
  const long long tiles = static_cast<long long>(a.groups) * ((a.M + tm - 1) / tm) * ((a.N + out_cols - 1) / out_cols);
  if (tiles <= 0) return MOE_OK;

#define MOE_GEMM_CASE(BN_, AMN_, BMN_, EPI_)                                               \
  if (a.bn == BN_ && a.a_mn == AMN_ && a.b_mn == BMN_ && a.epi == EPI_)                   \
    return a.pair ? launch_instance<BN_, AMN_, BMN_, EPI_, true>(maps, kp, tiles, st)     \
                  : launch_instance<BN_, AMN_, BMN_, EPI_, false>(maps, kp, tiles, st);
  // forward: projections / experts (bf16 out), SwiGLU, router logits, block output (f32)
  MOE_GEMM_CASE(256, false, false, EPI_BF16)
  MOE_GEMM_CASE(256, false, false, EPI_SWIGLU)
  MOE_GEMM_CASE(128, false, false, EPI_F32)
  MOE_GEMM_CASE(256, false, false, EPI_F32)
  if (a.bn == 192 && !a.a_mn && !a.b_mn && a.epi == EPI_F32 && a.pair)  // router logits, E % 192 == 0
    return launch_instance<192, false, false, EPI_F32, true>(maps, kp, tiles, st);
  // backward: dgrad (B stored [K][N]); dx in f32; wgrad (both stored [K][.]) in f32
  MOE_GEMM_CASE(256, false, true, EPI_BF16)
  MOE_GEMM_CASE(256, false, true, EPI_SWIGLU_BWD)
  MOE_GEMM_CASE(256, false, true, EPI_BF16_ADD_F32)
  MOE_GEMM_CASE(256, false, true, EPI_F32)
  // A stored [K][M] (MN-major): one CTA per tile only
#define MOE_GEMM_CASE1(BN_, AMN_, BMN_, EPI_)                                              \
  if (a.bn == BN_ && a.a_mn == AMN_ && a.b_mn == BMN_ && a.epi == EPI_ && !a.pair)        \
    return launch_instance<BN_, AMN_, BMN_, EPI_, false>(maps, kp, tiles, st);
  MOE_GEMM_CASE1(256, true, true, EPI_F32)
  // the remaining layouts of the test entry point
  MOE_GEMM_CASE1(256, true, false, EPI_F32)
  MOE_GEMM_CASE1(256, true, true, EPI_BF16)
  MOE_GEMM_CASE1(256, true, false, EPI_BF16)
#undef MOE_GEMM_CASE
#undef MOE_GEMM_CASE1
  return fail(MOE_ERR_UNSUPPORTED, "no gemm instance for this layout / epilogue");
}

}  // namespace moe
