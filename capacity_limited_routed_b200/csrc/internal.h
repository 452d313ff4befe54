// internal.h -- declarations shared by the translation units of libmoe (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <string>

#include "../../include/moe.h"

namespace moe {

// ------------------------------------------------------------------ errors

void set_error(const std::string& msg);
moe_status_t fail(moe_status_t code, const std::string& msg);
moe_status_t cuda_check(cudaError_t e, const char* what);

// ------------------------------------------------------------------ per-device set-up
//
// The CUDA runtime keeps function attributes (the dynamic shared-memory limit) and
// occupancy answers per device, so every cache of them is keyed by the device index.
// A set bit in a mask means "done on this device"; two threads racing on the same
// device only repeat the (idempotent) set-up.

constexpr int kMaxDevices = 64;

// index of the calling thread's current device, or -1 when there is none
int current_device();

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per device for `func`
moe_status_t ensure_max_smem(const void* func, int bytes, std::atomic<uint64_t>& done_mask, const char* what);

// ------------------------------------------------------------------ launch accounting

void count_launch(int n = 1);
int64_t launches_so_far();

// Brackets one step of a call with CUDA events while profiling is on.
class ProfScope {
 public:
  ProfScope(const char* name, cudaStream_t st);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;

 private:
  int slot_ = -1;
  cudaStream_t st_ = nullptr;
  int64_t launches0_ = 0;
};

// ------------------------------------------------------------------ GEMM

enum Epi : int {
  EPI_BF16 = 0,          // out = bf16(acc)
  EPI_F32 = 1,           // out = acc (+ col_add[col])
  EPI_SWIGLU = 2,        // acc = [gate | value]; out = bf16(silu(gate) * value); save_a/b = bf16(gate/value)
  EPI_SWIGLU_BWD = 3,    // acc = dH; out = dA = dH*b*silu'(a), out2 = dB = dH*silu(a)
  EPI_BF16_ADD_F32 = 4,  // out = bf16(acc + addend[row][col])
};

// A bf16 tensor in global memory seen as [groups][rows][inner], inner contiguous.
struct Mat {
  const void* ptr = nullptr;
  int64_t inner = 0, rows = 0, groups = 1;
  int64_t ld = 0;   // elements between consecutive rows (>= inner)
  int64_t gs = 0;   // elements between consecutive groups
};

// D[g][m][n] = sum over segments s, k of A_s(g, m, k) * B_s(g, n, k).
//   A K-major: A_s stored [M][K] (Mat inner = K);  A MN-major: stored [K][M] (inner = M).
//   B K-major: B_s stored [N][K];                  B MN-major: stored [K][N].
// ragged == 0: dense (or fixed-size groups).  ragged == 1: group g has
// group_rows[g] valid rows of M (tiles past them are skipped; rows up to M are
// stored).  ragged == 2: group g has group_rows[g] valid K (one segment; the
// operand's K extent zero-fills the rest).
struct GemmArgs {
  int bn = 256;
  bool pair = false;  // 256-row tiles on a pair of CTAs (cta_group::2); not with both operands MN-major
  bool a_mn = false, b_mn = false;
  int epi = EPI_BF16;
  int M = 0, N = 0;  // per group; N counts output columns
  int groups = 1;
  int ragged = 0;
  const int32_t* group_rows = nullptr;
  // ragged == 1 or 2 with buffers packed by expert: group g's rows start at row
  // group_off[g] of 2-D activation tensors (rows_total rows, groups = 1) instead of
  // being group g of a 3-D tensor; weights (and weight gradients) stay 3-D
  const int32_t* group_off = nullptr;
  int64_t rows_total = 0;
  int nseg = 1;
  Mat A[3], B[3];
  Mat Bv;            // value weights paired with B[0] for EPI_SWIGLU
  int64_t K[3] = {0, 0, 0};
  bool m_fastest = false;
  void* out = nullptr;
  int64_t ldo = 0, out_gs = 0;
  void* out2 = nullptr;
  void* save_a = nullptr;
  void* save_b = nullptr;
  const void* aux_a = nullptr;
  const void* aux_b = nullptr;
  int64_t aux_ld = 0, aux_gs = 0;
  const float* col_add = nullptr;
  const float* addend = nullptr;
  int64_t add_ld = 0;
  int32_t* status = nullptr;
  // launch group g is expert (g / map_p) * map_l + map_off + g % map_p (map_p = 0: g):
  // one wave's D * P experts as one launch; tensors stay indexed by expert and hold
  // tensor_groups groups (0: groups)
  int map_p = 0, map_l = 0, map_off = 0;
  int tensor_groups = 0;
};

moe_status_t gemm_run(const GemmArgs& a, cudaStream_t stream);
int device_sm_count();

// ------------------------------------------------------------------ routing / movement kernels

struct Geo {
  int T, E, k, D, W, L, P, NP, Cs, Cr, dl;
  int n_chunks;      // token chunks of the slot scan
  // virtual sources: T splits into S equal token ranges of Ts tokens (whole scan chunks),
  // each with its own D*W pools (NP of them) and sender caps; NPS = S * NP pools in all,
  // source-major.  S = 1 is one source.
  int S, Ts, NPS;
  // dropless variant: no cap binds (Cs = Cr = T*k); pools are packed back to back in
  // pool order (pool_rows = T*k rows) and expert buffers by expert, each expert's
  // region padded to a multiple of 128 rows (exp_rows = T*k + 127*E rows)
  bool dropless;
  int64_t pool_rows, exp_rows;
};

constexpr int kScanTokensPerChunk = 32;

// hist may be nullptr: the forward leaves the histogram to the slot scan (write_hist)
moe_status_t launch_route(const Geo& g, const float* logits, const float* bias, int32_t* idx, float* gate,
                          int32_t* hist, int32_t* nan_count, cudaStream_t st);
// scratch ints needed by the slot scan
size_t scan_scratch_ints(const Geo& g);
// write_hist: also write the selection histogram into the stats (every assignment's expert)
moe_status_t launch_slot_scan(const Geo& g, const int32_t* idx, int32_t* slot, int32_t* stats, int32_t* scratch,
                              cudaStream_t st, bool write_hist = false);
moe_status_t launch_pack(const Geo& g, const uint16_t* z, const int32_t* idx, const int32_t* slot,
                         int32_t* stats, uint16_t* pools, cudaStream_t st, const int32_t* pool_off = nullptr);
// off[i] = sum over j < i of round_up(counts[j], align), i = 0..n
moe_status_t launch_offsets(const int32_t* counts, int n, int align, int32_t* off, cudaStream_t st);
// scratch ints needed by the receiver's row map
size_t unpack_scratch_ints(const Geo& g);
// Receiver side: ranks the rows of every pool by their packed ids and copies the kept
// rows into the expert buffers xe.
// capacity layout: pool_off = exp_off = nullptr.  Dropless: pool_off / pool_fill give
// each pool's packed row range; exp_off (E+1 ints) is computed here from the counts.
// id_base: the packed (global) expert id of this receiver's expert 0 (expert parallelism)
moe_status_t launch_unpack(const Geo& g, const uint16_t* pools, uint16_t* xe, int32_t* rows, int32_t* row_map,
                           int32_t* status, cudaStream_t st, const int32_t* pool_off = nullptr,
                           const int32_t* pool_fill = nullptr, int32_t* exp_off = nullptr, int id_base = 0);
// rows between a receiver's pool positions and its expert rows by the row map (see map_rows_kernel)
moe_status_t launch_map_rows(const uint16_t* in, uint16_t* out, const int32_t* map, const uint16_t* hdr_pools,
                             int hdr_ld, int hdr_col, long long n_rows, int width, long long ld_pool, bool to_pools,
                             cudaStream_t st);
moe_status_t launch_zero_tail_rows(const Geo& g, uint16_t* buf, int64_t width, const int32_t* rows,
                                   cudaStream_t st, const int32_t* exp_off = nullptr);
// exp_off: row of each expert's first row in the expert buffers (dropless); nullptr:
// expert e's rows start at e * C_r.  by_pool: the expert rows are the ones receivers sent
// back under expert parallelism, laid out like the pools (row pool(e) * C_s + sender slot,
// receiver-dropped rows zero), and an assignment counts as kept when its sender kept it.
moe_status_t launch_combine(const Geo& g, const uint16_t* ye, const float* gate, const int32_t* idx,
                            const int32_t* slot, uint16_t* r, cudaStream_t st, const int32_t* exp_off = nullptr,
                            bool by_pool = false);
moe_status_t launch_combine_bwd(const Geo& g, const uint16_t* dr, const uint16_t* ye, const float* gate,
                                const int32_t* idx, const int32_t* slot, uint16_t* dye, float* dg,
                                cudaStream_t st, const int32_t* exp_off = nullptr, bool by_pool = false);
moe_status_t launch_undispatch(const Geo& g, const uint16_t* dxe, const float* gate, const float* dg,
                               const int32_t* idx, const int32_t* slot, float* dz_routed, uint16_t* dlogits,
                               cudaStream_t st, const int32_t* exp_off = nullptr, bool by_pool = false);
moe_status_t launch_bias_update(const Geo& g, const int32_t* hist, float* bias, float step, cudaStream_t st);
// out[i] = sum over s < S of part[s * n + i], float32, s in order (n a multiple of 4)
moe_status_t launch_sum_partials(const float* part, int S, long long n, float* out, cudaStream_t st);

// plan geometry and the device check, for entry points defined in other files
const Geo& plan_geo(const moe_plan* p);
moe_status_t device_check();

// stats buffer layout (int32 words)
constexpr int kStatsHead = 8;  // moe_stats_t
inline int stats_hist(const Geo& g) { return kStatsHead; }
inline int stats_kept_e(const Geo& g) { return kStatsHead + g.E; }
inline int stats_ds_e(const Geo& g) { return kStatsHead + 2 * g.E; }
inline int stats_dr_e(const Geo& g) { return kStatsHead + 3 * g.E; }
inline int stats_pool_fill(const Geo& g) { return kStatsHead + 4 * g.E; }
inline int stats_words(const Geo& g) { return kStatsHead + 4 * g.E + g.NPS; }

}  // namespace moe
