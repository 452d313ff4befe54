// moe_api.cu -- the C ABI of libmoe: plans, buffer layouts, argument checks and the order of
// launches for the forward and backward pass of the capacity-limited, pooled-wave MoE block.
//
// Step order of the forward pass ("Marin начинает открытое обучение MoE-модели с 535 млрд
// параметров", §2; "Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播", §2.2, §3.2):
// latent down-projection, router logits, top-k + gates + histogram, slot assignment,
// pack into pools (sender), unpack by packed id (receiver), grouped SwiGLU experts,
// combine, shared experts, up-projection fused with the shared down-projection.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

struct moe_plan {
  moe_config_t cfg;
  moe::Geo g;
  int dm, dl, E, k, h, S, hs;
  // forward context layout (byte offsets); training adds the SwiGLU pre-activations
  struct Ctx {
    size_t z, logits, idx, gate, slot, rows, xe, ae, be, he, ye, r, as, bs, hsh, exp_off, pool_off, bytes;
  } saved, infer;
  // scratch layouts
  size_t ws_scan, ws_pools, ws_rowmap, ws_ctx, ws_fwd_bytes;             // forward
  size_t ws_ffn_xe, ws_ffn_he, ws_ffn_rows, ws_ffn_rowmap, ws_ffn_bytes;  // moe_expert_ffn alone
  size_t b_dr, b_das, b_dbs, b_dye, b_dg, b_dae, b_dbe, b_dxe, b_dlog, b_dzr, b_dz, ws_bwd_bytes;
  size_t pools_bytes, expert_out_bytes, slot_bytes, stats_bytes, ws_bytes;
  // expert parallelism (G > 1): this rank is one source of T tokens (geometry g) and the
  // receiver of destinations [rank * D/G, ...), i.e. of E/G experts (geometry gr: G
  // sources, the same C_s, C_r from all ranks' tokens)
  int G, rank, E_loc;
  moe::Geo gr;
  struct Ep {
    // forward context: the source's, then the receiver's
    size_t z, logits, idx, gate, slot, r, as, bs, hsh, y_in;
    size_t recv_pools, xe, rows, row_map, ae, be, he, ye;
    size_t saved_bytes;
    // scratch: the exchange buffers, and what the backward keeps from its first call to its last
    size_t scan, send_pools, y_out, dy_out, dy_in, dx_out, dx_in;
    size_t dr, das, dbs, dg, dlog, dzr, dz;
    size_t dye, dae, dbe, dxe;
    size_t ws_bytes;
    size_t rows_bytes;  // one [D*W*C_s][d_latent] bf16 row buffer
  } ep;
};

namespace moe {

namespace {
thread_local std::string g_last_error;
thread_local const char* g_step = "";
}

void set_error(const std::string& msg) { g_last_error = msg; }

moe_status_t fail(moe_status_t code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

moe_status_t cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return MOE_OK;
  return fail(MOE_ERR_CUDA, std::string("[") + g_step + "] " + what + ": " + cudaGetErrorString(e));
}

// ---------------------------------------------------------------------- launch accounting

namespace {
std::atomic<int64_t> g_launches{0};

struct ProfRecord {
  char name[40];
  cudaEvent_t start, stop;
  int64_t launches;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRecord> g_prof;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
}  // namespace

void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
int64_t launches_so_far() { return g_launches.load(std::memory_order_relaxed); }

ProfScope::ProfScope(const char* name, cudaStream_t st) : st_(st) {
  g_step = name;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on) return;
  ProfRecord r;
  std::memset(&r, 0, sizeof(r));
  std::strncpy(r.name, name, sizeof(r.name) - 1);
  r.start = take_event();
  r.stop = take_event();
  if (r.start == nullptr || r.stop == nullptr) return;
  cudaEventRecord(r.start, st);
  launches0_ = launches_so_far();
  slot_ = static_cast<int>(g_prof.size());
  g_prof.push_back(r);
}

ProfScope::~ProfScope() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (slot_ >= static_cast<int>(g_prof.size())) return;
  cudaEventRecord(g_prof[slot_].stop, st_);
  g_prof[slot_].launches = launches_so_far() - launches0_;
}

}  // namespace moe

using namespace moe;

namespace {

constexpr size_t kAlign = 256;

size_t take(size_t& off, size_t bytes) {
  off = (off + kAlign - 1) / kAlign * kAlign;
  const size_t at = off;
  off += bytes;
  return at;
}

void layout_ctx(const moe_plan& p, bool training, moe_plan::Ctx& c) {
  // expert buffers: E x C_r rows, or (dropless) every assignment packed by expert with
  // each expert's region padded to 128 rows
  const size_t T = p.g.T, E = p.E, k = p.k, dl = p.dl, h = p.h, SH = size_t(p.S) * p.hs;
  const size_t R = size_t(p.g.exp_rows);
  size_t off = 0;
  c.z = take(off, T * dl * 2);
  c.logits = take(off, T * E * 4);
  c.idx = take(off, T * k * 4);
  c.gate = take(off, T * k * 4);
  c.slot = take(off, T * k * 8);
  c.rows = take(off, E * 4);
  c.xe = take(off, R * dl * 2);
  c.ae = training ? take(off, R * h * 2) : 0;
  c.be = training ? take(off, R * h * 2) : 0;
  c.he = take(off, R * h * 2);
  c.ye = take(off, R * dl * 2);
  c.r = take(off, T * dl * 2);
  c.as = training ? take(off, T * SH * 2) : 0;
  c.bs = training ? take(off, T * SH * 2) : 0;
  c.hsh = take(off, T * SH * 2);
  c.exp_off = take(off, (E + 1) * 4);
  c.pool_off = take(off, (size_t(p.g.NPS) + 1) * 4);
  c.bytes = (off + kAlign - 1) / kAlign * kAlign;
}

void layout(moe_plan& p) {
  const size_t T = p.g.T, E = p.E, k = p.k, dl = p.dl, h = p.h, SH = size_t(p.S) * p.hs;
  const size_t R = size_t(p.g.exp_rows);
  p.pools_bytes = size_t(p.g.pool_rows) * (dl + 8) * 2;
  layout_ctx(p, true, p.saved);
  layout_ctx(p, false, p.infer);
  p.expert_out_bytes = R * dl * 2;
  p.slot_bytes = T * k * 8;
  p.stats_bytes = size_t(stats_words(p.g)) * 4;
  size_t off = 0;
  p.ws_scan = take(off, scan_scratch_ints(p.g) * 4);
  p.ws_pools = take(off, p.pools_bytes);
  p.ws_rowmap = take(off, unpack_scratch_ints(p.g) * 4);
  p.ws_ctx = take(off, p.infer.bytes);  // used only when the forward keeps no context
  p.ws_fwd_bytes = off;
  off = 0;
  p.ws_ffn_xe = take(off, R * dl * 2);
  p.ws_ffn_he = take(off, R * h * 2);
  p.ws_ffn_rows = take(off, E * 4);
  p.ws_ffn_rowmap = take(off, unpack_scratch_ints(p.g) * 4);
  p.ws_ffn_bytes = off;
  off = 0;
  p.b_dr = take(off, T * dl * 2);
  p.b_das = take(off, T * SH * 2);
  p.b_dbs = take(off, T * SH * 2);
  p.b_dye = take(off, R * dl * 2);
  p.b_dg = take(off, T * k * 4);
  p.b_dae = take(off, R * h * 2);
  p.b_dbe = take(off, R * h * 2);
  p.b_dxe = take(off, R * dl * 2);
  p.b_dlog = take(off, T * E * 2);
  p.b_dzr = take(off, T * dl * 4);
  p.b_dz = take(off, T * dl * 2);
  p.ws_bwd_bytes = off;
  p.ws_bytes = std::max({p.ws_fwd_bytes, p.ws_ffn_bytes, p.ws_bwd_bytes, p.ws_scan + scan_scratch_ints(p.g) * 4});
  p.ws_bytes = (p.ws_bytes + kAlign - 1) / kAlign * kAlign;
}

// Layouts of an expert-parallel plan (see moe_plan::Ep).
void layout_ep(moe_plan& p) {
  const Geo& g = p.g;
  const Geo& r = p.gr;
  const size_t T = g.T, E = p.E, k = p.k, dl = p.dl, h = p.h, SH = size_t(p.S) * p.hs;
  const size_t prow = size_t(g.pool_rows);   // D*W*C_s: pools of this source = blocks a receiver gets
  const size_t Rr = size_t(r.exp_rows);      // E/G experts x C_r
  moe_plan::Ep& e = p.ep;
  e.rows_bytes = prow * dl * 2;
  size_t off = 0;
  e.z = take(off, T * dl * 2);
  e.logits = take(off, T * E * 4);
  e.idx = take(off, T * k * 4);
  e.gate = take(off, T * k * 4);
  e.slot = take(off, T * k * 8);
  e.r = take(off, T * dl * 2);
  e.as = take(off, T * SH * 2);
  e.bs = take(off, T * SH * 2);
  e.hsh = take(off, T * SH * 2);
  e.y_in = take(off, e.rows_bytes);
  e.recv_pools = take(off, p.pools_bytes);
  e.xe = take(off, Rr * dl * 2);
  e.rows = take(off, size_t(p.E_loc) * 4);
  e.row_map = take(off, prow * 4);
  e.ae = take(off, Rr * h * 2);
  e.be = take(off, Rr * h * 2);
  e.he = take(off, Rr * h * 2);
  e.ye = take(off, Rr * dl * 2);
  e.saved_bytes = (off + kAlign - 1) / kAlign * kAlign;
  off = 0;
  e.scan = take(off, scan_scratch_ints(g) * 4);
  e.send_pools = take(off, p.pools_bytes);
  e.y_out = take(off, e.rows_bytes);
  e.dy_out = take(off, e.rows_bytes);
  e.dy_in = take(off, e.rows_bytes);
  e.dx_out = take(off, e.rows_bytes);
  e.dx_in = take(off, e.rows_bytes);
  e.dr = take(off, T * dl * 2);
  e.das = take(off, T * SH * 2);
  e.dbs = take(off, T * SH * 2);
  e.dg = take(off, T * k * 4);
  e.dlog = take(off, T * E * 2);
  e.dzr = take(off, T * dl * 4);
  e.dz = take(off, T * dl * 2);
  e.dye = take(off, Rr * dl * 2);
  e.dae = take(off, Rr * h * 2);
  e.dbe = take(off, Rr * h * 2);
  e.dxe = take(off, Rr * dl * 2);
  e.ws_bytes = (off + kAlign - 1) / kAlign * kAlign;
}

// Capacities: expected rows times num/den, rounded up exactly (64-bit integers).
int32_t ceil_cap(int64_t rows_num, int64_t rows_den, int64_t num, int64_t den) {
  const int64_t a = rows_num * num, b = rows_den * den;
  return static_cast<int32_t>((a + b - 1) / b);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Once per device: is it an sm_100 part?
moe_status_t device_ok() {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MOE_ERR_UNSUPPORTED, std::string("no CUDA device: ") + cudaGetErrorString(e));
  }
  static std::atomic<int> checked[kMaxDevices];  // per device: 0 unknown, 1 ok, 2 bad
  if (dev >= 0 && dev < kMaxDevices && checked[dev].load(std::memory_order_relaxed) == 1) return MOE_OK;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) {
    if (dev >= 0 && dev < kMaxDevices) checked[dev].store(2, std::memory_order_relaxed);
    return fail(MOE_ERR_UNSUPPORTED, "libmoe needs an sm_100 (B200) device, found sm_" + std::to_string(major) +
                                         std::to_string(minor));
  }
  if (dev >= 0 && dev < kMaxDevices) checked[dev].store(1, std::memory_order_relaxed);
  return MOE_OK;
}

#define MOE_TRY(x)                       \
  do {                                   \
    moe_status_t _s = (x);               \
    if (_s != MOE_OK) return _s;         \
  } while (0)

// A second stream for the shared experts, which do not depend on routing: forked from the
// caller's stream by an event and joined back by another, so the routed path's short
// kernels can run beside the shared GEMMs.  One per host thread and device (a call's
// fork and join events are never recorded by another thread); created on first use.
// Stream capture of the caller's stream follows the fork into the side stream.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

std::atomic<int> g_use_side_stream{1};

// the side stream, or (moe_set_side_stream(0)) the caller's stream itself with no fork or join
moe_status_t side_stream(SideStream** out, cudaStream_t st) {
  if (g_use_side_stream.load(std::memory_order_relaxed) == 0) {
    thread_local SideStream inline_ss;
    inline_ss.s = st;
    inline_ss.fork = inline_ss.join = nullptr;
    *out = &inline_ss;
    return MOE_OK;
  }
  thread_local SideStream per_dev[kMaxDevices];
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device index out of range for the side stream");
  SideStream& ss = per_dev[dev];
  if (ss.s == nullptr) {
    MOE_TRY(cuda_check(cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking), "side stream"));
    MOE_TRY(cuda_check(cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming), "side stream fork event"));
    MOE_TRY(cuda_check(cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming), "side stream join event"));
  }
  *out = &ss;
  return MOE_OK;
}

// side stream waits for everything issued so far on st
moe_status_t fork_to(SideStream* ss, cudaStream_t st) {
  if (ss->fork == nullptr) return MOE_OK;  // the caller's stream itself
  MOE_TRY(cuda_check(cudaEventRecord(ss->fork, st), "fork record"));
  return cuda_check(cudaStreamWaitEvent(ss->s, ss->fork, 0), "fork wait");
}

// st waits for everything issued so far on the side stream
moe_status_t join_from(SideStream* ss, cudaStream_t st) {
  if (ss->join == nullptr) return MOE_OK;
  MOE_TRY(cuda_check(cudaEventRecord(ss->join, ss->s), "join record"));
  return cuda_check(cudaStreamWaitEvent(st, ss->join, 0), "join wait");
}

Mat mat(const void* ptr, int64_t inner, int64_t rows, int64_t groups = 1) {
  Mat m;
  m.ptr = ptr;
  m.inner = inner;
  m.rows = rows;
  m.groups = groups;
  m.ld = inner;
  m.gs = inner * rows;
  return m;
}

template <class T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}
template <class T>
const T* at(const void* base, size_t off) {
  return reinterpret_cast<const T*>(static_cast<const char*>(base) + off);
}

struct CtxPtrs {
  uint16_t *z, *xe, *ae, *be, *he, *ye, *r, *as, *bs, *hsh;
  float *logits, *gate;
  int32_t *idx, *slot, *rows;
  int32_t *exp_off, *pool_off;  // used by the dropless variant
};

CtxPtrs ctx_ptrs(const moe_plan& p, void* base, bool training) {
  const moe_plan::Ctx& c = training ? p.saved : p.infer;
  CtxPtrs q;
  q.z = at<uint16_t>(base, c.z);
  q.logits = at<float>(base, c.logits);
  q.idx = at<int32_t>(base, c.idx);
  q.gate = at<float>(base, c.gate);
  q.slot = at<int32_t>(base, c.slot);
  q.rows = at<int32_t>(base, c.rows);
  q.xe = at<uint16_t>(base, c.xe);
  q.ae = training ? at<uint16_t>(base, c.ae) : nullptr;
  q.be = training ? at<uint16_t>(base, c.be) : nullptr;
  q.he = at<uint16_t>(base, c.he);
  q.ye = at<uint16_t>(base, c.ye);
  q.r = at<uint16_t>(base, c.r);
  q.as = training ? at<uint16_t>(base, c.as) : nullptr;
  q.bs = training ? at<uint16_t>(base, c.bs) : nullptr;
  q.hsh = at<uint16_t>(base, c.hsh);
  q.exp_off = at<int32_t>(base, c.exp_off);
  q.pool_off = at<int32_t>(base, c.pool_off);
  return q;
}

// An expert activation buffer as a GEMM operand: E groups of C_r rows, or (dropless) one
// 2-D tensor of exp_rows rows whose group g starts at row exp_off[g].
Mat expert_mat(const Geo& g, const void* ptr, int64_t width) {
  return g.dropless ? mat(ptr, width, g.exp_rows, 1) : mat(ptr, width, g.Cr, g.E);
}

// Routed (ragged-row) GEMMs keep one CTA per 128-row tile: an expert's ~341 rows fill
// three of them (11% padding) but two 256-row pair tiles (50%), which measured slower.
void pack_groups(const Geo& g, GemmArgs& a, const int32_t* exp_off) {
  if (!g.dropless) return;
  a.group_off = exp_off;
  a.rows_total = g.exp_rows;
  if (a.ragged == 1) a.M = static_cast<int>(g.exp_rows);  // local rows never reach it
}

// Column tile of the router-logit GEMM (256-row pair tiles, N = E): 192 when it divides E
// and there are enough columns to matter, which turns E = 384 into two column tiles of a
// denser tile (128 pair tiles on 74 pairs) instead of three of 128.
int router_tile_cols(int E) { return (E >= 384 && E % 192 == 0) ? 192 : 128; }

// dW_r = dlogits^T z over the T tokens.  With K = T long and few output tiles (E x d_latent:
// 2 x 12 pair tiles at full width for 74 pairs) the tokens are split into S equal slices,
// computed as S groups of one launch into float32 partials in `scratch` (when it holds them)
// and summed in slice order.
moe_status_t router_wgrad(int E, int dl, int64_t T, const uint16_t* dlog, const uint16_t* z, float* out,
                          void* scratch, size_t scratch_bytes, cudaStream_t st) {
  const long long tiles = static_cast<long long>((E + 255) / 256) * ((dl + 255) / 256);
  int S = 1;
  for (int c = 4; c >= 2; c /= 2)
    if (T % c == 0 && T / c >= 1024 && tiles * c <= 2LL * device_sm_count() &&
        static_cast<size_t>(c) * E * dl * 4 <= scratch_bytes && (static_cast<long long>(E) * dl) % 4 == 0 &&
        (T / c) * E % 8 == 0 && (T / c) * dl % 8 == 0) {  // each slice 16-byte aligned
      S = c;
      break;
    }
  GemmArgs a;
  a.a_mn = a.b_mn = true;
  a.epi = EPI_F32;
  a.M = E;
  a.N = dl;
  a.ldo = dl;
  if (S == 1) {
    a.A[0] = mat(dlog, E, T);
    a.B[0] = mat(z, dl, T);
    a.K[0] = T;
    a.out = out;
    return gemm_run(a, st);
  }
  const int64_t Ts = T / S;
  a.groups = S;
  a.A[0] = mat(dlog, E, Ts, S);
  a.B[0] = mat(z, dl, Ts, S);
  a.K[0] = Ts;
  a.out = scratch;
  a.out_gs = static_cast<int64_t>(E) * dl;
  MOE_TRY(gemm_run(a, st));
  return launch_sum_partials(static_cast<const float*>(scratch), S, static_cast<long long>(E) * dl, out, st);
}

// receiver unpack + grouped SwiGLU experts (shared by moe_expert_ffn, moe_forward and the
// expert-parallel receiver): the receiver copies its kept rows into the expert buffers xe.
// g: the receiver's geometry; E its experts (weights [E][..]), dl, h the widths; id_base the
// packed (global) id of its expert 0.
moe_status_t run_experts_geo(const Geo& g, int E, int dl, int h, int id_base, const uint16_t* w1,
                             const uint16_t* w3, const uint16_t* w2, const uint16_t* pools, uint16_t* xe,
                             int32_t* rows, int32_t* row_map, uint16_t* ae, uint16_t* be, uint16_t* he,
                             uint16_t* ye, int32_t* status, cudaStream_t st, const int32_t* pool_off = nullptr,
                             const int32_t* pool_fill = nullptr, int32_t* exp_off = nullptr) {
  struct Dims {
    int E, dl, h;
  } p{E, dl, h};
  {
    ProfScope ps("experts.unpack", st);
    MOE_TRY(launch_unpack(g, pools, xe, rows, row_map, status, st, pool_off, pool_fill, exp_off, id_base));
    MOE_TRY(launch_zero_tail_rows(g, xe, dl, rows, st, exp_off));
  }
  // the three waves of identical shape, one after another: wave w is the D * P experts
  // with local index in [w * P, (w + 1) * P) of every destination
  for (int w = 0; w < g.W; ++w) {
    GemmArgs a;
    a.bn = 256;
    a.epi = EPI_SWIGLU;
    a.M = g.Cr;
    a.N = p.h;
    a.groups = g.D * g.P;
    a.map_p = g.P;
    a.map_l = g.L;
    a.map_off = w * g.P;
    a.tensor_groups = p.E;
    a.ragged = 1;
    a.group_rows = rows;
    a.A[0] = expert_mat(g, xe, p.dl);
    a.B[0] = mat(w1, p.dl, p.h, p.E);
    a.Bv = mat(w3, p.dl, p.h, p.E);
    a.K[0] = p.dl;
    a.m_fastest = true;
    a.out = he;
    a.ldo = p.h;
    a.out_gs = int64_t(g.Cr) * p.h;
    a.save_a = ae;
    a.save_b = be;
    a.status = status;
    pack_groups(g, a, exp_off);
    {
      ProfScope ps("experts.gate_up", st);
      MOE_TRY(gemm_run(a, st));
    }
    GemmArgs d;
    d.bn = 256;
    d.epi = EPI_BF16;
    d.M = g.Cr;
    d.N = p.dl;
    d.groups = g.D * g.P;
    d.map_p = g.P;
    d.map_l = g.L;
    d.map_off = w * g.P;
    d.tensor_groups = p.E;
    d.ragged = 1;
    d.group_rows = rows;
    d.A[0] = expert_mat(g, he, p.h);
    d.B[0] = mat(w2, p.h, p.dl, p.E);
    d.K[0] = p.h;
    d.m_fastest = true;
    d.out = ye;
    d.ldo = p.dl;
    d.out_gs = int64_t(g.Cr) * p.dl;
    d.status = status;
    pack_groups(g, d, exp_off);
    ProfScope ps("experts.down", st);
    MOE_TRY(gemm_run(d, st));
  }
  return MOE_OK;
}

moe_status_t run_experts(const moe_plan& p, const uint16_t* w1, const uint16_t* w3, const uint16_t* w2,
                         const uint16_t* pools, uint16_t* xe, int32_t* rows, int32_t* row_map, uint16_t* ae,
                         uint16_t* be, uint16_t* he, uint16_t* ye, int32_t* status, cudaStream_t st,
                         const int32_t* pool_off = nullptr, const int32_t* pool_fill = nullptr,
                         int32_t* exp_off = nullptr) {
  return run_experts_geo(p.g, p.E, p.dl, p.h, 0, w1, w3, w2, pools, xe, rows, row_map, ae, be, he, ye, status, st,
                         pool_off, pool_fill, exp_off);
}

// Backward of the routed experts on a receiver's rows, given dY (rows of dye):
// dH = dY w2 -> (dA, dB);  dw2 = dY^T H;  dX = dA w1 + dB w3;  dw1 = dA^T X, dw3 = dB^T X.
// g: the receiver's geometry, E its experts.
moe_status_t routed_backward(const Geo& g, int E, int dl, int h, const uint16_t* w1, const uint16_t* w3,
                             const uint16_t* w2, const int32_t* rows, const uint16_t* xe, const uint16_t* ae, const uint16_t* be, const uint16_t* he, const uint16_t* dye,
                             uint16_t* dae, uint16_t* dbe, uint16_t* dxe, float* gw1, float* gw3, float* gw2,
                             cudaStream_t st, const int32_t* exp_off) {
  const int64_t Cr = g.Cr;
  {
    ProfScope ps("bwd.experts_dgrad_down", st);
    GemmArgs a;
    a.b_mn = true;
    a.epi = EPI_SWIGLU_BWD;
    a.M = g.Cr;
    a.N = h;
    a.groups = E;
    a.ragged = 1;
    a.group_rows = rows;
    a.A[0] = expert_mat(g, dye, dl);
    a.B[0] = mat(w2, h, dl, E);
    a.K[0] = dl;
    a.m_fastest = true;
    a.aux_a = ae;
    a.aux_b = be;
    a.aux_ld = h;
    a.aux_gs = Cr * h;
    a.out = dae;
    a.out2 = dbe;
    a.ldo = h;
    a.out_gs = Cr * h;
    pack_groups(g, a, exp_off);
    MOE_TRY(gemm_run(a, st));
  }
  {
    ProfScope ps("bwd.experts_wgrad_down", st);
    GemmArgs a;
    a.a_mn = a.b_mn = true;
    a.epi = EPI_F32;
    a.M = dl;
    a.N = h;
    a.groups = E;
    a.ragged = 2;
    a.group_rows = rows;
    a.m_fastest = false;  // concurrent tiles write whole rows of dW
    a.A[0] = expert_mat(g, dye, dl);
    a.B[0] = expert_mat(g, he, h);
    a.out = gw2;
    a.ldo = h;
    a.out_gs = int64_t(dl) * h;
    pack_groups(g, a, exp_off);
    MOE_TRY(gemm_run(a, st));
  }
  {
    ProfScope ps("bwd.experts_dgrad_gate_up", st);
    GemmArgs a;
    a.b_mn = true;
    a.M = g.Cr;
    a.N = dl;
    a.groups = E;
    a.ragged = 1;
    a.group_rows = rows;
    a.nseg = 2;
    a.A[0] = expert_mat(g, dae, h);
    a.B[0] = mat(w1, dl, h, E);
    a.K[0] = h;
    a.A[1] = expert_mat(g, dbe, h);
    a.B[1] = mat(w3, dl, h, E);
    a.K[1] = h;
    a.m_fastest = true;
    a.out = dxe;
    a.ldo = dl;
    a.out_gs = Cr * dl;
    pack_groups(g, a, exp_off);
    MOE_TRY(gemm_run(a, st));
  }
  {
    ProfScope ps("bwd.experts_wgrad_gate_up", st);
    GemmArgs a;
    a.a_mn = a.b_mn = true;
    a.epi = EPI_F32;
    a.M = h;
    a.N = dl;
    a.groups = E;
    a.ragged = 2;
    a.group_rows = rows;
    a.m_fastest = false;  // concurrent tiles write whole rows of dW
    a.A[0] = expert_mat(g, dae, h);
    a.B[0] = expert_mat(g, xe, dl);
    a.out = gw1;
    a.ldo = dl;
    a.out_gs = int64_t(h) * dl;
    pack_groups(g, a, exp_off);
    MOE_TRY(gemm_run(a, st));
    a.A[0] = expert_mat(g, dbe, h);
    a.out = gw3;
    MOE_TRY(gemm_run(a, st));
  }
  return MOE_OK;
}

}  // namespace

namespace moe {
const Geo& plan_geo(const moe_plan* p) { return p->g; }
moe_status_t device_check() { return device_ok(); }
}  // namespace moe

extern "C" {

const char* moe_last_error(void) { return g_last_error.c_str(); }

moe_status_t moe_profile_start(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof) {
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  g_prof.clear();
  g_prof_on = true;
  return MOE_OK;
}

moe_status_t moe_profile_stop(moe_profile_record_t* out, int32_t cap, int32_t* count) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = false;
  int32_t n = 0;
  for (auto& r : g_prof) {
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return cuda_check(cudaGetLastError(), "profile sync");
    if (out != nullptr && n < cap) {
      std::memcpy(out[n].name, r.name, sizeof(out[n].name));
      float ms = 0.0f;
      cudaEventElapsedTime(&ms, r.start, r.stop);
      out[n].ms = ms;
      out[n].launches = static_cast<int32_t>(r.launches);
    }
    ++n;
  }
  if (count != nullptr) *count = n;
  return MOE_OK;
}

int64_t moe_kernel_launches(void) { return launches_so_far(); }

moe_status_t moe_set_side_stream(int32_t side_stream) {
  if (side_stream != 0 && side_stream != 1) return fail(MOE_ERR_INVALID_ARG, "side_stream must be 0 or 1");
  g_use_side_stream.store(side_stream, std::memory_order_relaxed);
  return MOE_OK;
}

moe_status_t moe_plan_create(const moe_config_t* cfg, moe_plan_t* out) {
  if (cfg == nullptr || out == nullptr) return fail(MOE_ERR_INVALID_ARG, "null argument");
  *out = nullptr;
  const moe_config_t& c = *cfg;
  if (c.T < 0 || c.d_model <= 0 || c.d_latent <= 0 || c.n_experts <= 0 || c.top_k <= 0 || c.n_dest <= 0 ||
      c.n_waves <= 0 || c.hidden_routed <= 0 || c.n_shared <= 0 || c.hidden_shared <= 0)
    return fail(MOE_ERR_INVALID_ARG, "sizes must be positive (T may be 0)");
  // both numerators 0: the dropless variant (no cap binds)
  const bool dropless = c.cap_send_num == 0 && c.cap_recv_num == 0;
  if (!dropless && (c.cap_send_num <= 0 || c.cap_send_den <= 0 || c.cap_recv_num <= 0 || c.cap_recv_den <= 0))
    return fail(MOE_ERR_INVALID_ARG, "capacity ratios must be positive (or both numerators 0: dropless)");
  if (c.n_experts % c.n_dest != 0) return fail(MOE_ERR_UNSUPPORTED, "E must be a multiple of D");
  const int L = c.n_experts / c.n_dest;
  if (L % c.n_waves != 0) return fail(MOE_ERR_UNSUPPORTED, "E/D must be a multiple of the wave count");
  if (c.top_k > c.n_experts || c.top_k > 32) return fail(MOE_ERR_UNSUPPORTED, "top_k must be <= min(E, 32)");
  if (c.n_experts > 1024 || c.n_experts % 8 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "E must be a multiple of 8, at most 1024");
  if (c.d_model % 64 || c.d_latent % 64) return fail(MOE_ERR_UNSUPPORTED, "d_model and d_latent must be multiples of 64");
  if (c.hidden_routed % 128 || c.hidden_shared % 128)
    return fail(MOE_ERR_UNSUPPORTED, "hidden widths must be multiples of 128");
  if (L / c.n_waves > 32) return fail(MOE_ERR_UNSUPPORTED, "at most 32 experts per wave");
  const int64_t A = int64_t(c.T) * c.top_k;
  if (A > (int64_t(1) << 30)) return fail(MOE_ERR_UNSUPPORTED, "T * top_k too large");
  // virtual sources (0 reads as 1): each source's tokens are whole chunks of the slot scan
  const int S = c.n_sources > 0 ? c.n_sources : 1;
  if (c.n_sources < 0) return fail(MOE_ERR_INVALID_ARG, "n_sources must be >= 0");
  if (S > 1 && (c.T % S != 0 || (c.T / S) % kScanTokensPerChunk != 0))
    return fail(MOE_ERR_UNSUPPORTED, "with several sources T/S must be a multiple of " +
                                         std::to_string(kScanTokensPerChunk));
  // expert parallelism: G ranks, each one source and the receiver of D/G destinations
  const int G = c.ep_ranks > 1 ? c.ep_ranks : 1;
  if (c.ep_ranks < 0) return fail(MOE_ERR_INVALID_ARG, "ep_ranks must be >= 0");
  if (G > 1) {
    if (c.ep_rank < 0 || c.ep_rank >= G) return fail(MOE_ERR_INVALID_ARG, "ep_rank must be in [0, ep_ranks)");
    if (c.n_dest % G != 0) return fail(MOE_ERR_UNSUPPORTED, "expert parallelism needs D a multiple of the ranks");
    if (S > 1) return fail(MOE_ERR_UNSUPPORTED, "under expert parallelism every rank is one source");
    if (dropless) return fail(MOE_ERR_UNSUPPORTED, "expert parallelism runs the capped variant");
  }
  moe_plan* p = new moe_plan();
  std::memset(static_cast<void*>(p), 0, sizeof(*p));
  p->cfg = c;
  p->dm = c.d_model;
  p->dl = c.d_latent;
  p->E = c.n_experts;
  p->k = c.top_k;
  p->h = c.hidden_routed;
  p->S = c.n_shared;
  p->hs = c.hidden_shared;
  Geo& g = p->g;
  g.T = c.T;
  g.E = c.n_experts;
  g.k = c.top_k;
  g.D = c.n_dest;
  g.W = c.n_waves;
  g.L = L;
  g.P = L / c.n_waves;
  g.NP = c.n_dest * c.n_waves;
  g.S = S;
  g.Ts = S > 1 ? c.T / S : (c.T > 0 ? c.T : 1);
  g.NPS = S * g.NP;
  g.dropless = dropless;
  if (dropless) {
    // no slot reaches T*k, so no cap binds; buffers are packed (see Geo)
    g.Cs = g.Cr = static_cast<int32_t>(A > 0 ? A : 1);
    g.pool_rows = A;
    g.exp_rows = A + int64_t(127) * c.n_experts;
  } else {
    // a source's pool expects (T/S)*k/(D*W) rows
    g.Cs = ceil_cap(A, int64_t(c.n_dest) * c.n_waves * S, c.cap_send_num, c.cap_send_den);
    g.Cr = ceil_cap(A, c.n_experts, c.cap_recv_num, c.cap_recv_den);
    if (g.Cs < 1) g.Cs = 1;
    if (g.Cr < 1) g.Cr = 1;
    g.pool_rows = int64_t(g.NPS) * g.Cs;
    g.exp_rows = int64_t(c.n_experts) * g.Cr;
  }
  g.dl = c.d_latent;
  g.n_chunks = (c.T + kScanTokensPerChunk - 1) / kScanTokensPerChunk;
  if (g.n_chunks < 1) g.n_chunks = 1;
  p->G = G;
  p->rank = G > 1 ? c.ep_rank : 0;
  p->E_loc = c.n_experts / G;
  if (G > 1) {
    // every rank's tokens reach the receivers: C_r from all G * T of them
    g.Cr = std::max(1, ceil_cap(int64_t(G) * A, c.n_experts, c.cap_recv_num, c.cap_recv_den));
    g.exp_rows = int64_t(c.n_experts) * g.Cr;
    Geo& r = p->gr;
    r = g;
    r.E = p->E_loc;
    r.D = c.n_dest / G;
    r.NP = r.D * r.W;
    r.S = G;              // the G sources' pools, source-major
    r.Ts = c.T;
    r.NPS = G * r.NP;     // = D * W: as many pools as one source sends
    r.pool_rows = int64_t(r.NPS) * r.Cs;
    r.exp_rows = int64_t(r.E) * r.Cr;
  }
  layout(*p);
  if (G > 1) layout_ep(*p);
  *out = p;
  return MOE_OK;
}

moe_status_t moe_plan_destroy(moe_plan_t plan) {
  delete plan;
  return MOE_OK;
}

moe_status_t moe_plan_info(moe_plan_t p, moe_plan_info_t* out) {
  if (p == nullptr || out == nullptr) return fail(MOE_ERR_INVALID_ARG, "null argument");
  out->local_experts = p->g.L;
  out->experts_per_wave = p->g.P;
  out->n_pools = p->g.NPS;  // every source's D*W pools, source-major
  out->cap_send = p->g.dropless ? 0 : p->g.Cs;  // 0: no cap (dropless)
  out->cap_recv = p->g.dropless ? 0 : p->g.Cr;
  out->pool_row_elems = p->dl + 8;
  out->pools_bytes = p->pools_bytes;
  out->expert_out_bytes = p->expert_out_bytes;
  out->slot_bytes = p->slot_bytes;
  out->stats_bytes = p->stats_bytes;
  out->saved_bytes = p->G > 1 ? p->ep.saved_bytes : p->saved.bytes;
  out->workspace_bytes = p->G > 1 ? p->ep.ws_bytes : p->ws_bytes;
  return MOE_OK;
}

moe_status_t moe_saved_view(moe_plan_t p, const void* saved, moe_saved_view_t* out) {
  if (p == nullptr || saved == nullptr || out == nullptr) return fail(MOE_ERR_INVALID_ARG, "null argument");
  CtxPtrs q = ctx_ptrs(*p, const_cast<void*>(saved), true);
  out->z = q.z;
  out->logits = q.logits;
  out->topk_idx = q.idx;
  out->topk_gate = q.gate;
  out->slot = q.slot;
  out->expert_rows = q.rows;
  out->expert_in = q.xe;
  out->expert_out = q.ye;
  out->r = q.r;
  return MOE_OK;
}

moe_status_t moe_route(moe_plan_t p, const float* logits, const float* bias, int32_t* topk_idx, float* topk_gate,
                       int32_t* hist, void* stream) {
  if (p == nullptr) return fail(MOE_ERR_INVALID_ARG, "null plan");
  if (p->g.T > 0 && (!logits || !topk_idx || !topk_gate)) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  if (!bias || !hist) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  MOE_TRY(device_ok());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_TRY(cuda_check(cudaMemsetAsync(hist, 0, sizeof(int32_t) * p->E, st), "hist memset"));
  return launch_route(p->g, logits, bias, topk_idx, topk_gate, hist, nullptr, st);
}

moe_status_t moe_dispatch(moe_plan_t p, const uint16_t* z, const int32_t* topk_idx, uint16_t* pools, int32_t* slot,
                          void* stats, void* ws, size_t ws_bytes, void* stream) {
  if (p == nullptr) return fail(MOE_ERR_INVALID_ARG, "null plan");
  if (p->g.dropless)
    return fail(MOE_ERR_UNSUPPORTED, "the dropless variant runs through moe_forward / moe_backward only");
  if (!pools || !stats || !ws) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  if (p->g.T > 0 && (!z || !topk_idx || !slot)) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  if (!aligned16(z) || !aligned16(pools)) return fail(MOE_ERR_INVALID_ARG, "z and pools must be 16-byte aligned");
  if (ws_bytes < p->ws_scan + scan_scratch_ints(p->g) * 4) return fail(MOE_ERR_WORKSPACE, "workspace too small");
  MOE_TRY(device_ok());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* s = static_cast<int32_t*>(stats);
  MOE_TRY(launch_slot_scan(p->g, topk_idx, slot, s, at<int32_t>(ws, p->ws_scan), st));
  return launch_pack(p->g, z, topk_idx, slot, s, pools, st);
}

moe_status_t moe_expert_ffn(moe_plan_t p, const moe_expert_weights_t* w, const uint16_t* pools, uint16_t* expert_out,
                            int32_t* expert_rows, void* ws, size_t ws_bytes, void* stream) {
  if (p == nullptr || w == nullptr) return fail(MOE_ERR_INVALID_ARG, "null argument");
  if (p->g.dropless)
    return fail(MOE_ERR_UNSUPPORTED, "the dropless variant runs through moe_forward / moe_backward only");
  if (!w->w1 || !w->w3 || !w->w2 || !pools || !expert_out || !ws)
    return fail(MOE_ERR_INVALID_ARG, "null buffer");
  if (p->G > 1) return fail(MOE_ERR_UNSUPPORTED, "an expert-parallel plan runs through the moe_ep_* calls");
  if (ws_bytes < p->ws_ffn_bytes) return fail(MOE_ERR_WORKSPACE, "workspace too small");
  if (!aligned16(expert_out)) return fail(MOE_ERR_INVALID_ARG, "expert_out must be 16-byte aligned");
  MOE_TRY(device_ok());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* rows = expert_rows ? expert_rows : at<int32_t>(ws, p->ws_ffn_rows);
  return run_experts(*p, w->w1, w->w3, w->w2, pools, at<uint16_t>(ws, p->ws_ffn_xe), rows,
                     at<int32_t>(ws, p->ws_ffn_rowmap), nullptr, nullptr, at<uint16_t>(ws, p->ws_ffn_he), expert_out,
                     nullptr, st);
}

moe_status_t moe_combine(moe_plan_t p, const uint16_t* expert_out, const float* topk_gate, const int32_t* topk_idx,
                         const int32_t* slot, uint16_t* r, void* stream) {
  if (p == nullptr) return fail(MOE_ERR_INVALID_ARG, "null plan");
  if (p->g.dropless)
    return fail(MOE_ERR_UNSUPPORTED, "the dropless variant runs through moe_forward / moe_backward only");
  if (p->G > 1) return fail(MOE_ERR_UNSUPPORTED, "an expert-parallel plan runs through the moe_ep_* calls");
  if (p->g.T == 0) return MOE_OK;
  if (!expert_out || !topk_gate || !topk_idx || !slot || !r) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  if (!aligned16(expert_out) || !aligned16(r)) return fail(MOE_ERR_INVALID_ARG, "buffers must be 16-byte aligned");
  MOE_TRY(device_ok());
  return launch_combine(p->g, expert_out, topk_gate, topk_idx, slot, r, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_forward(moe_plan_t p, const moe_weights_t* w, const uint16_t* x, const float* bias,
                         const float* logit_offset, float* y, void* stats, void* saved, void* ws, size_t ws_bytes,
                         void* stream) {
  if (p == nullptr || w == nullptr) return fail(MOE_ERR_INVALID_ARG, "null argument");
  if (!w->w_lat_down || !w->w_router || !w->w1 || !w->w3 || !w->w2 || !w->w_lat_up || !w->ws1 || !w->ws3 ||
      !w->ws2)
    return fail(MOE_ERR_INVALID_ARG, "null weight");
  if (!bias || !stats || !ws) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  if (p->g.T > 0 && (!x || !y)) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  if (p->G > 1) return fail(MOE_ERR_UNSUPPORTED, "an expert-parallel plan runs through the moe_ep_* calls");
  if (ws_bytes < p->ws_fwd_bytes) return fail(MOE_ERR_WORKSPACE, "workspace too small");
  MOE_TRY(device_ok());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* s = static_cast<int32_t*>(stats);
  const Geo& g = p->g;
  MOE_TRY(cuda_check(cudaMemsetAsync(s, 0, p->stats_bytes, st), "stats memset"));
  if (g.T == 0) return MOE_OK;
  const bool training = saved != nullptr;
  CtxPtrs c = ctx_ptrs(*p, training ? saved : at<void>(ws, p->ws_ctx), training);
  int32_t* status = s + 3;
  const int64_t SH = int64_t(p->S) * p->hs;

  // latent down-projection: z = x W_lat_down^T
  {
    ProfScope ps("fwd.lat_down", st);
    GemmArgs a;
    a.pair = true;  // dense rows: 256-row tiles on CTA pairs
    a.M = g.T;
    a.N = p->dl;
    a.A[0] = mat(x, p->dm, g.T);
    a.B[0] = mat(w->w_lat_down, p->dm, p->dl);
    a.K[0] = p->dm;
    a.out = c.z;
    a.ldo = p->dl;
    a.status = status;
    MOE_TRY(gemm_run(a, st));
  }
  // router logits (float32, + per-expert offset)
  {
    ProfScope ps("fwd.router", st);
    GemmArgs a;
    a.pair = true;  // dense rows: 256-row tiles on CTA pairs
    a.bn = router_tile_cols(p->E);
    a.epi = EPI_F32;
    a.M = g.T;
    a.N = p->E;
    a.A[0] = mat(c.z, p->dl, g.T);
    a.B[0] = mat(w->w_router, p->dl, p->E);
    a.K[0] = p->dl;
    a.out = c.logits;
    a.ldo = p->E;
    a.col_add = logit_offset;
    a.status = status;
    MOE_TRY(gemm_run(a, st));
  }
  // shared experts on the side stream, beside the routing, movement and expert kernels:
  // H_s = silu(x ws1^T) * (x ws3^T)
  SideStream* ss = nullptr;
  MOE_TRY(side_stream(&ss, st));
  MOE_TRY(fork_to(ss, st));
  {
    ProfScope ps("fwd.shared_gate_up", ss->s);
    GemmArgs a;
    a.pair = true;  // dense rows: 256-row tiles on CTA pairs
    a.epi = EPI_SWIGLU;
    a.M = g.T;
    a.N = static_cast<int>(SH);
    a.A[0] = mat(x, p->dm, g.T);
    a.B[0] = mat(w->ws1, p->dm, SH);
    a.Bv = mat(w->ws3, p->dm, SH);
    a.K[0] = p->dm;
    a.out = c.hsh;
    a.ldo = SH;
    a.save_a = c.as;
    a.save_b = c.bs;
    a.status = status;
    MOE_TRY(gemm_run(a, ss->s));
  }

  {
    ProfScope ps("fwd.route_topk", st);
    MOE_TRY(launch_route(g, c.logits, bias, c.idx, c.gate, nullptr, s + 7, st));
  }
  {
    ProfScope ps("fwd.slot_scan", st);  // also the selection histogram
    MOE_TRY(launch_slot_scan(g, c.idx, c.slot, s, at<int32_t>(ws, p->ws_scan), st, true));
  }
  uint16_t* pools = at<uint16_t>(ws, p->ws_pools);
  // dropless: pools and expert buffers are packed; their offsets come from the counts
  int32_t* pool_off = g.dropless ? c.pool_off : nullptr;
  int32_t* exp_off = g.dropless ? c.exp_off : nullptr;
  {
    ProfScope ps("fwd.dispatch_pack", st);
    if (g.dropless) MOE_TRY(launch_offsets(s + stats_pool_fill(g), g.NPS, 1, pool_off, st));
    MOE_TRY(launch_pack(g, c.z, c.idx, c.slot, s, pools, st, pool_off));
  }
  MOE_TRY(run_experts(*p, w->w1, w->w3, w->w2, pools, c.xe, c.rows, at<int32_t>(ws, p->ws_rowmap), c.ae, c.be,
                      c.he, c.ye, status, st, pool_off, g.dropless ? s + stats_pool_fill(g) : nullptr, exp_off));
  {
    ProfScope ps("fwd.combine", st);
    MOE_TRY(launch_combine(g, c.ye, c.gate, c.idx, c.slot, c.r, st, exp_off));
  }
  MOE_TRY(join_from(ss, st));
  // y = r W_lat_up^T + H_s ws2^T (two K segments, one accumulator), float32 out
  {
    ProfScope ps("fwd.lat_up_shared_down", st);
    GemmArgs a;
    a.pair = true;  // dense rows: 256-row tiles on CTA pairs
    a.epi = EPI_F32;
    a.M = g.T;
    a.N = p->dm;
    a.nseg = 2;
    a.A[0] = mat(c.r, p->dl, g.T);
    a.B[0] = mat(w->w_lat_up, p->dl, p->dm);
    a.K[0] = p->dl;
    a.A[1] = mat(c.hsh, SH, g.T);
    a.B[1] = mat(w->ws2, SH, p->dm);
    a.K[1] = SH;
    a.out = y;
    a.ldo = p->dm;
    a.status = status;
    MOE_TRY(gemm_run(a, st));
  }
  return MOE_OK;
}

moe_status_t moe_backward(moe_plan_t p, const moe_weights_t* w, const void* saved, const uint16_t* x,
                          const uint16_t* dy, float* dx, const moe_grads_t* gr, void* ws, size_t ws_bytes,
                          void* stream) {
  if (p == nullptr || w == nullptr || gr == nullptr) return fail(MOE_ERR_INVALID_ARG, "null argument");
  if (!saved || !ws) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  if (!w->w_lat_down || !w->w_router || !w->w1 || !w->w3 || !w->w2 || !w->w_lat_up || !w->ws1 || !w->ws3 ||
      !w->ws2)
    return fail(MOE_ERR_INVALID_ARG, "null weight");
  if (!gr->w_lat_down || !gr->w_router || !gr->w1 || !gr->w3 || !gr->w2 || !gr->w_lat_up || !gr->ws1 || !gr->ws3 ||
      !gr->ws2)
    return fail(MOE_ERR_INVALID_ARG, "null gradient");
  if (p->g.T > 0 && (!x || !dy || !dx)) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  if (p->G > 1) return fail(MOE_ERR_UNSUPPORTED, "an expert-parallel plan runs through the moe_ep_* calls");
  if (ws_bytes < p->ws_bwd_bytes) return fail(MOE_ERR_WORKSPACE, "workspace too small");
  MOE_TRY(device_ok());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Geo& g = p->g;
  const int64_t SH = int64_t(p->S) * p->hs;
  const int64_t T = g.T, E = p->E, Cr = g.Cr, dl = p->dl, dm = p->dm, h = p->h;
  if (g.T == 0) {
    // no tokens: every gradient is zero
    const size_t sizes[9] = {size_t(dl * dm), size_t(E * dl), size_t(E * h * dl), size_t(E * h * dl),
                             size_t(E * dl * h), size_t(dm * dl), size_t(SH * dm), size_t(SH * dm), size_t(dm * SH)};
    float* ptrs[9] = {gr->w_lat_down, gr->w_router, gr->w1, gr->w3, gr->w2, gr->w_lat_up, gr->ws1, gr->ws3, gr->ws2};
    for (int i = 0; i < 9; ++i) MOE_TRY(cuda_check(cudaMemsetAsync(ptrs[i], 0, sizes[i] * 4, st), "grad memset"));
    return MOE_OK;
  }
  CtxPtrs c = ctx_ptrs(*p, const_cast<void*>(saved), true);
  const int32_t* exp_off = g.dropless ? c.exp_off : nullptr;  // packed expert buffers (dropless)
  uint16_t* dr = at<uint16_t>(ws, p->b_dr);
  uint16_t* das = at<uint16_t>(ws, p->b_das);
  uint16_t* dbs = at<uint16_t>(ws, p->b_dbs);
  uint16_t* dye = at<uint16_t>(ws, p->b_dye);
  float* dg = at<float>(ws, p->b_dg);
  uint16_t* dae = at<uint16_t>(ws, p->b_dae);
  uint16_t* dbe = at<uint16_t>(ws, p->b_dbe);
  uint16_t* dxe = at<uint16_t>(ws, p->b_dxe);
  uint16_t* dlog = at<uint16_t>(ws, p->b_dlog);
  float* dzr = at<float>(ws, p->b_dzr);
  uint16_t* dz = at<uint16_t>(ws, p->b_dz);
  int32_t* status = nullptr;

  // y = r W_up^T + H_s ws2^T:  dr = dy W_up,  dH_s = dy ws2 -> SwiGLU backward
  {
    ProfScope ps("bwd.dr", st);
    GemmArgs a;
    a.pair = true;  // dense rows: 256-row tiles on CTA pairs
    a.b_mn = true;
    a.M = g.T;
    a.N = p->dl;
    a.A[0] = mat(dy, dm, T);
    a.B[0] = mat(w->w_lat_up, dl, dm);
    a.K[0] = dm;
    a.out = dr;
    a.ldo = dl;
    MOE_TRY(gemm_run(a, st));
  }
  // dW_up = dy^T r
  {
    ProfScope ps("bwd.wgrad_lat_up", st);
    GemmArgs a;
    a.a_mn = a.b_mn = true;
    a.epi = EPI_F32;
    a.M = static_cast<int>(dm);
    a.N = static_cast<int>(dl);
    a.A[0] = mat(dy, dm, T);
    a.B[0] = mat(c.r, dl, T);
    a.K[0] = T;
    a.out = gr->w_lat_up;
    a.ldo = dl;
    MOE_TRY(gemm_run(a, st));
  }
  // combine backward: dY = g dr on kept rows, dg = <dr, Y>
  {
    ProfScope ps("bwd.combine", st);
    MOE_TRY(launch_combine_bwd(g, dr, c.ye, c.gate, c.idx, c.slot, dye, dg, st, exp_off));
    MOE_TRY(launch_zero_tail_rows(g, dye, dl, c.rows, st, exp_off));
  }
  MOE_TRY(routed_backward(g, static_cast<int>(E), static_cast<int>(dl), static_cast<int>(h), w->w1, w->w3, w->w2,
                          c.rows, c.xe, c.ae, c.be, c.he, dye, dae, dbe, dxe, gr->w1, gr->w3, gr->w2, st,
                          exp_off));
  // the shared experts' backward on the side stream, beside un-dispatch and the router's
  // backward (joined before dx): dH_s = dy ws2 -> SwiGLU backward -> (dA_s, dB_s);
  // dws2 = dy^T H_s;  dws1 = dA_s^T x, dws3 = dB_s^T x
  SideStream* ss = nullptr;
  MOE_TRY(side_stream(&ss, st));
  MOE_TRY(fork_to(ss, st));
  {
    ProfScope ps("bwd.shared_dgrad_swiglu", ss->s);
    GemmArgs a;
    a.pair = true;  // dense rows: 256-row tiles on CTA pairs
    a.b_mn = true;
    a.epi = EPI_SWIGLU_BWD;
    a.M = g.T;
    a.N = static_cast<int>(SH);
    a.A[0] = mat(dy, dm, T);
    a.B[0] = mat(w->ws2, SH, dm);
    a.K[0] = dm;
    a.aux_a = c.as;
    a.aux_b = c.bs;
    a.aux_ld = SH;
    a.out = das;
    a.out2 = dbs;
    a.ldo = SH;
    MOE_TRY(gemm_run(a, ss->s));
  }
  {
    ProfScope ps("bwd.wgrad_shared", ss->s);
    GemmArgs a;
    a.a_mn = a.b_mn = true;
    a.epi = EPI_F32;
    a.M = static_cast<int>(dm);
    a.N = static_cast<int>(SH);
    a.A[0] = mat(dy, dm, T);
    a.B[0] = mat(c.hsh, SH, T);
    a.K[0] = T;
    a.out = gr->ws2;
    a.ldo = SH;
    MOE_TRY(gemm_run(a, ss->s));
    a.M = static_cast<int>(SH);
    a.N = static_cast<int>(dm);
    a.B[0] = mat(x, dm, T);
    a.ldo = dm;
    a.A[0] = mat(das, SH, T);
    a.out = gr->ws1;
    MOE_TRY(gemm_run(a, ss->s));
    a.A[0] = mat(dbs, SH, T);
    a.out = gr->ws3;
    MOE_TRY(gemm_run(a, ss->s));
  }
  // un-dispatch and the softmax backward to the logits
  {
    ProfScope ps("bwd.undispatch", st);
    MOE_TRY(launch_undispatch(g, dxe, c.gate, dg, c.idx, c.slot, dzr, dlog, st, exp_off));
  }
  // dz = dlogits W_r + dz_routed;  dW_r = dlogits^T z
  {
    ProfScope ps("bwd.router_dgrad", st);
    GemmArgs a;
    a.pair = true;  // dense rows: 256-row tiles on CTA pairs
    a.b_mn = true;
    a.epi = EPI_BF16_ADD_F32;
    a.M = g.T;
    a.N = static_cast<int>(dl);
    a.A[0] = mat(dlog, E, T);
    a.B[0] = mat(w->w_router, dl, E);
    a.K[0] = E;
    a.addend = dzr;
    a.add_ld = dl;
    a.out = dz;
    a.ldo = dl;
    MOE_TRY(gemm_run(a, st));
  }
  {
    // the routed backward's dA buffer is free again here: it holds the split's partials
    ProfScope ps("bwd.router_wgrad", st);
    MOE_TRY(router_wgrad(static_cast<int>(E), static_cast<int>(dl), T, dlog, c.z, gr->w_router, dae,
                         p->b_dbe - p->b_dae, st));
  }
  MOE_TRY(join_from(ss, st));
  // dx = dz W_down + dA_s ws1 + dB_s ws3 (three K segments), float32 out
  {
    ProfScope ps("bwd.dx", st);
    GemmArgs a;
    a.pair = true;  // dense rows: 256-row tiles on CTA pairs
    a.epi = EPI_F32;
    a.b_mn = true;
    a.M = g.T;
    a.N = static_cast<int>(dm);
    a.nseg = 3;
    a.A[0] = mat(dz, dl, T);
    a.B[0] = mat(w->w_lat_down, dm, dl);
    a.K[0] = dl;
    a.A[1] = mat(das, SH, T);
    a.B[1] = mat(w->ws1, dm, SH);
    a.K[1] = SH;
    a.A[2] = mat(dbs, SH, T);
    a.B[2] = mat(w->ws3, dm, SH);
    a.K[2] = SH;
    a.out = dx;
    a.ldo = dm;
    MOE_TRY(gemm_run(a, st));
  }
  // dW_down = dz^T x
  {
    ProfScope ps("bwd.wgrad_lat_down", st);
    GemmArgs a;
    a.a_mn = a.b_mn = true;
    a.epi = EPI_F32;
    a.M = static_cast<int>(dl);
    a.N = static_cast<int>(dm);
    a.A[0] = mat(dz, dl, T);
    a.B[0] = mat(x, dm, T);
    a.K[0] = T;
    a.out = gr->w_lat_down;
    a.ldo = dm;
    MOE_TRY(gemm_run(a, st));
  }
  (void)status;
  return MOE_OK;
}

moe_status_t moe_bias_update(moe_plan_t p, const int32_t* hist, float* bias, float step, void* stream) {
  if (p == nullptr || !hist || !bias) return fail(MOE_ERR_INVALID_ARG, "null argument");
  MOE_TRY(device_ok());
  ProfScope ps("bias_update", static_cast<cudaStream_t>(stream));
  return launch_bias_update(p->g, hist, bias, step, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_gemm_bf16(int32_t M, int32_t N, int32_t K, const uint16_t* A, int32_t a_mn_major, const uint16_t* B,
                           int32_t b_mn_major, void* D, int32_t d_f32, int32_t* status, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0) return fail(MOE_ERR_INVALID_ARG, "sizes must be positive");
  if (!A || !B || !D) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  const int64_t a_inner = a_mn_major ? M : K, b_inner = b_mn_major ? N : K;
  if (a_inner % 8 || b_inner % 8 || N % 8)
    return fail(MOE_ERR_UNSUPPORTED, "contiguous dimensions and N must be multiples of 8");
  MOE_TRY(device_ok());
  GemmArgs a;
  a.a_mn = a_mn_major != 0;
  a.b_mn = b_mn_major != 0;
  a.pair = !a.a_mn && M > 128;  // as the block's dense GEMMs run (A stored [M][K])
  a.epi = d_f32 ? EPI_F32 : EPI_BF16;
  a.M = M;
  a.N = N;
  a.A[0] = a.a_mn ? mat(A, M, K) : mat(A, K, M);
  a.B[0] = a.b_mn ? mat(B, N, K) : mat(B, K, N);
  a.K[0] = K;
  a.out = D;
  a.ldo = N;
  a.status = status;
  return gemm_run(a, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ====================================================================== expert parallelism

namespace {

struct EpPtrs {
  uint16_t *z, *r, *as, *bs, *hsh, *y_in, *recv_pools, *xe, *ae, *be, *he, *ye;
  float *logits, *gate;
  int32_t *idx, *slot, *rows, *row_map;
  int32_t* scan;
  uint16_t *send_pools, *y_out, *dy_out, *dy_in, *dx_out, *dx_in, *dr, *das, *dbs, *dlog, *dz;
  float *dg, *dzr;
  uint16_t *dye, *dae, *dbe, *dxe;
};

EpPtrs ep_ptrs(const moe_plan& p, const void* saved, void* ws) {
  const moe_plan::Ep& e = p.ep;
  EpPtrs q;
  void* sv = const_cast<void*>(saved);
  q.z = at<uint16_t>(sv, e.z);
  q.logits = at<float>(sv, e.logits);
  q.idx = at<int32_t>(sv, e.idx);
  q.gate = at<float>(sv, e.gate);
  q.slot = at<int32_t>(sv, e.slot);
  q.r = at<uint16_t>(sv, e.r);
  q.as = at<uint16_t>(sv, e.as);
  q.bs = at<uint16_t>(sv, e.bs);
  q.hsh = at<uint16_t>(sv, e.hsh);
  q.y_in = at<uint16_t>(sv, e.y_in);
  q.recv_pools = at<uint16_t>(sv, e.recv_pools);
  q.xe = at<uint16_t>(sv, e.xe);
  q.rows = at<int32_t>(sv, e.rows);
  q.row_map = at<int32_t>(sv, e.row_map);
  q.ae = at<uint16_t>(sv, e.ae);
  q.be = at<uint16_t>(sv, e.be);
  q.he = at<uint16_t>(sv, e.he);
  q.ye = at<uint16_t>(sv, e.ye);
  q.scan = at<int32_t>(ws, e.scan);
  q.send_pools = at<uint16_t>(ws, e.send_pools);
  q.y_out = at<uint16_t>(ws, e.y_out);
  q.dy_out = at<uint16_t>(ws, e.dy_out);
  q.dy_in = at<uint16_t>(ws, e.dy_in);
  q.dx_out = at<uint16_t>(ws, e.dx_out);
  q.dx_in = at<uint16_t>(ws, e.dx_in);
  q.dr = at<uint16_t>(ws, e.dr);
  q.das = at<uint16_t>(ws, e.das);
  q.dbs = at<uint16_t>(ws, e.dbs);
  q.dg = at<float>(ws, e.dg);
  q.dlog = at<uint16_t>(ws, e.dlog);
  q.dzr = at<float>(ws, e.dzr);
  q.dz = at<uint16_t>(ws, e.dz);
  q.dye = at<uint16_t>(ws, e.dye);
  q.dae = at<uint16_t>(ws, e.dae);
  q.dbe = at<uint16_t>(ws, e.dbe);
  q.dxe = at<uint16_t>(ws, e.dxe);
  return q;
}

moe_status_t ep_check(const moe_plan* p, const void* saved, const void* ws, size_t ws_bytes) {
  if (p == nullptr) return fail(MOE_ERR_INVALID_ARG, "null plan");
  if (p->G < 2) return fail(MOE_ERR_UNSUPPORTED, "the moe_ep_* calls need a plan with ep_ranks >= 2");
  if (saved == nullptr || ws == nullptr) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  if (ws_bytes < p->ep.ws_bytes) return fail(MOE_ERR_WORKSPACE, "workspace too small");
  return device_ok();
}

}  // namespace

extern "C" {

moe_status_t moe_ep_view(moe_plan_t p, void* saved, void* ws, moe_ep_view_t* out) {
  if (p == nullptr || out == nullptr || saved == nullptr || ws == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "null argument");
  if (p->G < 2) return fail(MOE_ERR_UNSUPPORTED, "not an expert-parallel plan");
  EpPtrs q = ep_ptrs(*p, saved, ws);
  out->ranks = p->G;
  out->rank = p->rank;
  out->dest_per_rank = p->gr.D;
  out->n_waves = p->g.W;
  out->cap_send = p->g.Cs;
  out->pool_row_elems = p->dl + 8;
  out->row_elems = p->dl;
  out->send_pools = q.send_pools;
  out->recv_pools = q.recv_pools;
  out->y_send = q.y_out;
  out->y_recv = q.y_in;
  out->dy_send = q.dy_out;
  out->dy_recv = q.dy_in;
  out->dx_send = q.dx_out;
  out->dx_recv = q.dx_in;
  out->expert_rows = q.rows;
  out->topk_idx = q.idx;
  out->slot = q.slot;
  return MOE_OK;
}

moe_status_t moe_ep_forward_send(moe_plan_t p, const moe_weights_t* w, const uint16_t* x, const float* bias,
                                 const float* logit_offset, void* stats, void* saved, void* ws, size_t ws_bytes,
                                 void* stream) {
  MOE_TRY(ep_check(p, saved, ws, ws_bytes));
  if (w == nullptr || !w->w_lat_down || !w->w_router || !w->ws1 || !w->ws3) return fail(MOE_ERR_INVALID_ARG, "null weight");
  if (!bias || !stats || (p->g.T > 0 && !x)) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Geo& g = p->g;
  int32_t* s = static_cast<int32_t*>(stats);
  EpPtrs c = ep_ptrs(*p, saved, ws);
  MOE_TRY(cuda_check(cudaMemsetAsync(s, 0, p->stats_bytes, st), "stats memset"));
  int32_t* status = s + 3;
  const int64_t SH = int64_t(p->S) * p->hs;
  SideStream* ss = nullptr;
  MOE_TRY(side_stream(&ss, st));
  MOE_TRY(fork_to(ss, st));
  if (g.T > 0) {
    ProfScope ps("fwd.shared_gate_up", ss->s);
    GemmArgs a;
    a.pair = true;  // dense rows: 256-row tiles on CTA pairs
    a.epi = EPI_SWIGLU;
    a.M = g.T;
    a.N = static_cast<int>(SH);
    a.A[0] = mat(x, p->dm, g.T);
    a.B[0] = mat(w->ws1, p->dm, SH);
    a.Bv = mat(w->ws3, p->dm, SH);
    a.K[0] = p->dm;
    a.out = c.hsh;
    a.ldo = SH;
    a.save_a = c.as;
    a.save_b = c.bs;
    a.status = status;
    MOE_TRY(gemm_run(a, ss->s));
  }
  if (g.T > 0) {
    {
      ProfScope ps("fwd.lat_down", st);
      GemmArgs a;
      a.pair = true;
      a.M = g.T;
      a.N = p->dl;
      a.A[0] = mat(x, p->dm, g.T);
      a.B[0] = mat(w->w_lat_down, p->dm, p->dl);
      a.K[0] = p->dm;
      a.out = c.z;
      a.ldo = p->dl;
      a.status = status;
      MOE_TRY(gemm_run(a, st));
    }
    {
      ProfScope ps("fwd.router", st);
      GemmArgs a;
      a.pair = true;
      a.bn = router_tile_cols(p->E);
      a.epi = EPI_F32;
      a.M = g.T;
      a.N = p->E;
      a.A[0] = mat(c.z, p->dl, g.T);
      a.B[0] = mat(w->w_router, p->dl, p->E);
      a.K[0] = p->dl;
      a.out = c.logits;
      a.ldo = p->E;
      a.col_add = logit_offset;
      a.status = status;
      MOE_TRY(gemm_run(a, st));
    }
    {
      ProfScope ps("fwd.route_topk", st);
      MOE_TRY(launch_route(g, c.logits, bias, c.idx, c.gate, nullptr, s + 7, st));
    }
    {
      ProfScope ps("fwd.slot_scan", st);  // also the selection histogram
      MOE_TRY(launch_slot_scan(g, c.idx, c.slot, s, c.scan, st, true));
    }
  }
  {
    ProfScope ps("fwd.dispatch_pack", st);
    MOE_TRY(launch_pack(g, c.z, c.idx, c.slot, s, c.send_pools, st));
  }
  return join_from(ss, st);
}

moe_status_t moe_ep_forward_experts(moe_plan_t p, const moe_expert_weights_t* ew, void* stats, void* saved, void* ws,
                                    size_t ws_bytes, void* stream) {
  MOE_TRY(ep_check(p, saved, ws, ws_bytes));
  if (ew == nullptr || !ew->w1 || !ew->w3 || !ew->w2 || !stats) return fail(MOE_ERR_INVALID_ARG, "null argument");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Geo& r = p->gr;
  EpPtrs c = ep_ptrs(*p, saved, ws);
  int32_t* status = static_cast<int32_t*>(stats) + 3;
  MOE_TRY(run_experts_geo(r, p->E_loc, p->dl, p->h, p->rank * p->E_loc, ew->w1, ew->w3, ew->w2, c.recv_pools, c.xe,
                          c.rows, c.row_map, c.ae, c.be, c.he, c.ye, status, st));
  ProfScope ps("experts.return", st);
  return launch_map_rows(c.ye, c.y_out, c.row_map, c.recv_pools, p->dl + 8, p->dl, r.pool_rows, p->dl, p->dl,
                         true, st);
}

moe_status_t moe_ep_forward_combine(moe_plan_t p, const moe_weights_t* w, float* y, void* saved, void* ws,
                                    size_t ws_bytes, void* stream) {
  MOE_TRY(ep_check(p, saved, ws, ws_bytes));
  if (w == nullptr || !w->w_lat_up || !w->ws2) return fail(MOE_ERR_INVALID_ARG, "null weight");
  const Geo& g = p->g;
  if (g.T == 0) return MOE_OK;
  if (!y) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  EpPtrs c = ep_ptrs(*p, saved, ws);
  const int64_t SH = int64_t(p->S) * p->hs;
  {
    ProfScope ps("fwd.combine", st);
    MOE_TRY(launch_combine(g, c.y_in, c.gate, c.idx, c.slot, c.r, st, nullptr, true));
  }
  ProfScope ps("fwd.lat_up_shared_down", st);
  GemmArgs a;
  a.pair = true;
  a.epi = EPI_F32;
  a.M = g.T;
  a.N = p->dm;
  a.nseg = 2;
  a.A[0] = mat(c.r, p->dl, g.T);
  a.B[0] = mat(w->w_lat_up, p->dl, p->dm);
  a.K[0] = p->dl;
  a.A[1] = mat(c.hsh, SH, g.T);
  a.B[1] = mat(w->ws2, SH, p->dm);
  a.K[1] = SH;
  a.out = y;
  a.ldo = p->dm;
  return gemm_run(a, st);
}

moe_status_t moe_ep_backward_send(moe_plan_t p, const moe_weights_t* w, const void* saved, const uint16_t* x,
                                  const uint16_t* dy, const moe_grads_t* gr, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(ep_check(p, saved, ws, ws_bytes));
  if (w == nullptr || gr == nullptr || !w->w_lat_up || !w->ws2 || !gr->w_lat_up || !gr->ws1 || !gr->ws3 || !gr->ws2)
    return fail(MOE_ERR_INVALID_ARG, "null argument");
  const Geo& g = p->g;
  const int64_t SH = int64_t(p->S) * p->hs, T = g.T, dl = p->dl, dm = p->dm;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    float* ptrs[4] = {gr->w_lat_up, gr->ws1, gr->ws3, gr->ws2};
    const size_t sizes[4] = {size_t(dm * dl), size_t(SH * dm), size_t(SH * dm), size_t(dm * SH)};
    for (int i = 0; i < 4; ++i) MOE_TRY(cuda_check(cudaMemsetAsync(ptrs[i], 0, sizes[i] * 4, st), "grad memset"));
    return MOE_OK;
  }
  if (!x || !dy) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  EpPtrs c = ep_ptrs(*p, saved, ws);
  SideStream* ss = nullptr;
  MOE_TRY(side_stream(&ss, st));
  MOE_TRY(fork_to(ss, st));
  {
    ProfScope ps("bwd.shared_dgrad_swiglu", ss->s);
    GemmArgs a;
    a.pair = true;
    a.b_mn = true;
    a.epi = EPI_SWIGLU_BWD;
    a.M = g.T;
    a.N = static_cast<int>(SH);
    a.A[0] = mat(dy, dm, T);
    a.B[0] = mat(w->ws2, SH, dm);
    a.K[0] = dm;
    a.aux_a = c.as;
    a.aux_b = c.bs;
    a.aux_ld = SH;
    a.out = c.das;
    a.out2 = c.dbs;
    a.ldo = SH;
    MOE_TRY(gemm_run(a, ss->s));
  }
  {
    ProfScope ps("bwd.wgrad_shared", ss->s);
    GemmArgs a;
    a.a_mn = a.b_mn = true;
    a.epi = EPI_F32;
    a.M = static_cast<int>(dm);
    a.N = static_cast<int>(SH);
    a.A[0] = mat(dy, dm, T);
    a.B[0] = mat(c.hsh, SH, T);
    a.K[0] = T;
    a.out = gr->ws2;
    a.ldo = SH;
    MOE_TRY(gemm_run(a, ss->s));
    a.M = static_cast<int>(SH);
    a.N = static_cast<int>(dm);
    a.B[0] = mat(x, dm, T);
    a.ldo = dm;
    a.A[0] = mat(c.das, SH, T);
    a.out = gr->ws1;
    MOE_TRY(gemm_run(a, ss->s));
    a.A[0] = mat(c.dbs, SH, T);
    a.out = gr->ws3;
    MOE_TRY(gemm_run(a, ss->s));
  }
  {
    ProfScope ps("bwd.dr", st);
    GemmArgs a;
    a.pair = true;
    a.b_mn = true;
    a.M = g.T;
    a.N = p->dl;
    a.A[0] = mat(dy, dm, T);
    a.B[0] = mat(w->w_lat_up, dl, dm);
    a.K[0] = dm;
    a.out = c.dr;
    a.ldo = dl;
    MOE_TRY(gemm_run(a, st));
  }
  {
    ProfScope ps("bwd.wgrad_lat_up", st);
    GemmArgs a;
    a.a_mn = a.b_mn = true;
    a.epi = EPI_F32;
    a.M = static_cast<int>(dm);
    a.N = static_cast<int>(dl);
    a.A[0] = mat(dy, dm, T);
    a.B[0] = mat(c.r, dl, T);
    a.K[0] = T;
    a.out = gr->w_lat_up;
    a.ldo = dl;
    MOE_TRY(gemm_run(a, st));
  }
  {
    // dY = g dr at the pool positions of the sender-kept rows, dg = <dr, Y> with the rows
    // the receivers returned (zeros for the ones they dropped)
    ProfScope ps("bwd.combine", st);
    MOE_TRY(launch_combine_bwd(g, c.dr, c.y_in, c.gate, c.idx, c.slot, c.dy_out, c.dg, st, nullptr, true));
  }
  return join_from(ss, st);
}

moe_status_t moe_ep_backward_experts(moe_plan_t p, const moe_expert_weights_t* ew, const void* saved,
                                     const moe_grads_t* gr, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(ep_check(p, saved, ws, ws_bytes));
  if (ew == nullptr || gr == nullptr || !ew->w1 || !ew->w3 || !ew->w2 || !gr->w1 || !gr->w3 || !gr->w2)
    return fail(MOE_ERR_INVALID_ARG, "null argument");
  const Geo& r = p->gr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  EpPtrs c = ep_ptrs(*p, saved, ws);
  {
    // the received dY rows into the expert buffers (receiver-kept rows only)
    ProfScope ps("bwd.combine", st);
    MOE_TRY(launch_map_rows(c.dy_in, c.dye, c.row_map, nullptr, 0, 0, r.pool_rows, p->dl, p->dl, false, st));
    MOE_TRY(launch_zero_tail_rows(r, c.dye, p->dl, c.rows, st));
  }
  MOE_TRY(routed_backward(r, p->E_loc, p->dl, p->h, ew->w1, ew->w3, ew->w2, c.rows, c.xe, c.ae, c.be, c.he, c.dye,
                          c.dae, c.dbe, c.dxe, gr->w1, gr->w3, gr->w2, st, nullptr));
  ProfScope ps("bwd.experts_return", st);
  return launch_map_rows(c.dxe, c.dx_out, c.row_map, c.recv_pools, p->dl + 8, p->dl, r.pool_rows, p->dl, p->dl, true,
                         st);
}

moe_status_t moe_ep_backward_finish(moe_plan_t p, const moe_weights_t* w, const void* saved, const uint16_t* x,
                                    float* dx, const moe_grads_t* gr, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(ep_check(p, saved, ws, ws_bytes));
  if (w == nullptr || gr == nullptr || !w->w_lat_down || !w->w_router || !w->ws1 || !w->ws3 || !gr->w_lat_down ||
      !gr->w_router)
    return fail(MOE_ERR_INVALID_ARG, "null argument");
  const Geo& g = p->g;
  const int64_t SH = int64_t(p->S) * p->hs, T = g.T, dl = p->dl, dm = p->dm, E = p->E;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    MOE_TRY(cuda_check(cudaMemsetAsync(gr->w_lat_down, 0, size_t(dl * dm) * 4, st), "grad memset"));
    return cuda_check(cudaMemsetAsync(gr->w_router, 0, size_t(E * dl) * 4, st), "grad memset");
  }
  if (!x || !dx) return fail(MOE_ERR_INVALID_ARG, "null buffer");
  EpPtrs c = ep_ptrs(*p, saved, ws);
  const size_t dae_bytes = p->ep.dbe - p->ep.dae;
  {
    ProfScope ps("bwd.undispatch", st);
    MOE_TRY(launch_undispatch(g, c.dx_in, c.gate, c.dg, c.idx, c.slot, c.dzr, c.dlog, st, nullptr, true));
  }
  {
    ProfScope ps("bwd.router_dgrad", st);
    GemmArgs a;
    a.pair = true;
    a.b_mn = true;
    a.epi = EPI_BF16_ADD_F32;
    a.M = g.T;
    a.N = static_cast<int>(dl);
    a.A[0] = mat(c.dlog, E, T);
    a.B[0] = mat(w->w_router, dl, E);
    a.K[0] = E;
    a.addend = c.dzr;
    a.add_ld = dl;
    a.out = c.dz;
    a.ldo = dl;
    MOE_TRY(gemm_run(a, st));
  }
  {
    // the receiver's dA buffer is free again here: it holds the split's partials
    ProfScope ps("bwd.router_wgrad", st);
    MOE_TRY(router_wgrad(static_cast<int>(E), static_cast<int>(dl), T, c.dlog, c.z, gr->w_router, c.dae,
                         dae_bytes, st));
  }
  {
    ProfScope ps("bwd.dx", st);
    GemmArgs a;
    a.pair = true;
    a.epi = EPI_F32;
    a.b_mn = true;
    a.M = g.T;
    a.N = static_cast<int>(dm);
    a.nseg = 3;
    a.A[0] = mat(c.dz, dl, T);
    a.B[0] = mat(w->w_lat_down, dm, dl);
    a.K[0] = dl;
    a.A[1] = mat(c.das, SH, T);
    a.B[1] = mat(w->ws1, dm, SH);
    a.K[1] = SH;
    a.A[2] = mat(c.dbs, SH, T);
    a.B[2] = mat(w->ws3, dm, SH);
    a.K[2] = SH;
    a.out = dx;
    a.ldo = dm;
    MOE_TRY(gemm_run(a, st));
  }
  ProfScope ps("bwd.wgrad_lat_down", st);
  GemmArgs a;
  a.a_mn = a.b_mn = true;
  a.epi = EPI_F32;
  a.M = static_cast<int>(dl);
  a.N = static_cast<int>(dm);
  a.A[0] = mat(c.dz, dl, T);
  a.B[0] = mat(x, dm, T);
  a.K[0] = T;
  a.out = gr->w_lat_down;
  a.ldo = dm;
  return gemm_run(a, st);
}

}  // extern "C"
