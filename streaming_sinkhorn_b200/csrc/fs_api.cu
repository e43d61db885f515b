// fs_api.cu -- the C ABI (include/fs.h): argument checks, input validation on the device,
// workspace carving, launch planning and stream ordering of the streaming passes.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/fs.h"
#include "fs_screen.cuh"
#include "fs_transport.cuh"
#include "fs_tc.cuh"
#include "fs_tc_wide.cuh"
#include "fs_small.cuh"

namespace fs {
namespace {

thread_local char g_cuda_err[256] = "";
std::atomic<int64_t> g_launches{0};
// Error bits the next call ORs into its error word (fs_inject_error_word), 0 = none.
std::atomic<unsigned> g_inject{0};

struct CudaFail {};

inline void ck(cudaError_t e, const char* what) {
  if (e != cudaSuccess) {
    snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", what, cudaGetErrorString(e));
    throw CudaFail{};
  }
}
#define CK(call) ck((call), #call)

// ---------------- kernel timing ----------------
std::mutex g_timing_mu;
bool g_timing_on = false;
std::atomic<bool> g_screening{true};
fs_timing g_timing = {};

enum TimedKind { kTLse = 0, kTGrad = 1, kTMarg = 2, kTCombine = 3, kTScreen = 4 };

struct TimedLaunch {
  cudaEvent_t start, stop;
  int kind;
  double pairs;
};

class Timer {
 public:
  explicit Timer(cudaStream_t s) : stream_(s) {
    std::lock_guard<std::mutex> lk(g_timing_mu);
    on_ = g_timing_on;
  }
  ~Timer() {
    for (auto& t : rec_) {
      cudaEventDestroy(t.start);
      cudaEventDestroy(t.stop);
    }
  }
  bool on() const { return on_; }
  int begin() {
    if (!on_) return -1;
    TimedLaunch t{};
    CK(cudaEventCreate(&t.start));
    CK(cudaEventCreate(&t.stop));
    CK(cudaEventRecord(t.start, stream_));
    rec_.push_back(t);
    return static_cast<int>(rec_.size()) - 1;
  }
  void end(int idx, int kind, double pairs) {
    if (idx < 0) return;
    rec_[idx].kind = kind;
    rec_[idx].pairs = pairs;
    CK(cudaEventRecord(rec_[idx].stop, stream_));
  }
  // Call after the stream has been synchronised; `evaluated[k]` = pairs the sorted passes
  // of timed kind k evaluated in this call after screening.
  void collect(const unsigned long long* evaluated) {
    if (!on_) return;
    std::lock_guard<std::mutex> lk(g_timing_mu);
    g_timing.lse_pass.evaluated += static_cast<double>(evaluated[kTLse]);
    g_timing.grad_pass.evaluated += static_cast<double>(evaluated[kTGrad]);
    g_timing.marg_pass.evaluated += static_cast<double>(evaluated[kTMarg]);
    for (auto& t : rec_) {
      float ms = 0.f;
      CK(cudaEventElapsedTime(&ms, t.start, t.stop));
      fs_timing_entry* e = t.kind == kTLse    ? &g_timing.lse_pass
                           : t.kind == kTGrad ? &g_timing.grad_pass
                           : t.kind == kTMarg ? &g_timing.marg_pass
                           : t.kind == kTScreen ? &g_timing.screen
                                              : &g_timing.combine;
      e->launches += 1;
      e->total_ms += ms;
      e->pairs += t.pairs;
    }
  }

 private:
  cudaStream_t stream_;
  bool on_ = false;
  std::vector<TimedLaunch> rec_;
};

// ---------------- shapes, plans and the workspace ----------------

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

int padded_dim(int d) {
  if (d <= 4) return d;
  if (d <= 8) return 8;
  if (d <= 16) return 16;
  if (d <= 32) return 32;
  return 64;
}

int64_t pairs_pad(int64_t count) { return round_up(ceil_div(count, 2), kPairPad); }

// Launch variants of the streaming pass. Index 0 has the most rows per CTA; the planner
// falls back to index 1 only for problems too small to fill the GPU otherwise.
//   D <= 16, potential/marginal passes: (R, NT, G, min CTAs/SM) = (2, 128, 8, 6), (1, 128, 8, 8)
//   D <= 16, gradient passes:                                   (2, 128, 8, 3), (1, 128, 8, 4)
//   D > 16, every pass:                                          (1, 128, 4, 1)
// (2 rows per thread at 6 CTAs/SM measured fastest among 1-8 rows x 128-512 threads.)
struct Variant {
  int R, NT;
};
// d <= 16: one warp per CTA over 64 rows, so each warp centres, streams (and, screened,
// screens and merges) on its own and never waits at a barrier for another warp's tiles.
constexpr Variant kNarrowVariant = {2, 32};
constexpr int kNarrowStages = 2;  // one tile in flight while one is consumed
// d > 16 (the gradient pass of wide points): four warps share each tile.
constexpr Variant kWideVariant = {1, 128};
constexpr int kQueueVariant = 0;
constexpr Variant kQueueShape = kNarrowVariant;
constexpr int kQueueStages = kNarrowStages;
inline int stages_for(int D) { return D > 16 ? kStages : kNarrowStages; }

struct Plan {
  int variant;  // index into the variant table of this pass type
  int R, NT;
  int64_t n_rows;
  int64_t row_blocks, rows_pad;
  int tile_pairs;
  int n_splits;
  int64_t pairs_per_split;
};

int num_sms_current() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaGetLastError();
  return sms > 0 ? sms : 148;
}

// The copy ring of key tiles and, for the screened passes of D <= 3 (which skip 16-point
// groups), one slot of group records behind it.
size_t pass_smem_bytes(int D, int tile_pairs, int stages = kStages, int np = 0,
                       bool group_recs = false) {
  const size_t ring = static_cast<size_t>(stages) * tile_pairs * pair_floats(D, np);
  return (ring + (group_recs && D <= 3 ? static_cast<size_t>(kTileGroupFloats) : 0u)) * 4;
}

// Pass kernel selector: what the pass accumulates (PassMode) and, for transport products,
// how many payload channels its key tiles carry.
enum PassSel : int { kSelLse = 0, kSelGrad = 1, kSelPay1 = 2, kSelPay4 = 3, kSelPay16 = 4,
                     kSelDiff = 5 };

// defined after the kernels; queue: the screened launches' kernel
int occupancy_for(int D, bool grad, int variant, size_t smem, bool queue = false);

Plan make_plan(int64_t n_rows, int64_t key_pairs, int D, bool grad, int sms) {
  const int64_t fill = static_cast<int64_t>(sms) * (D > 16 ? 4 : 16);
  const int max_tile = D > 16 ? 32 : 128;
  const Variant* vars = D > 16 ? &kWideVariant : &kNarrowVariant;
  const int nv = 1;
  Plan p{};
  p.n_rows = n_rows;
  // Most rows per CTA whose (row blocks x tiles) still fills the machine; else the smallest.
  int chosen = nv - 1;
  for (int v = 0; v < nv; ++v) {
    const int64_t rb = ceil_div(n_rows, static_cast<int64_t>(vars[v].R) * vars[v].NT);
    if (rb * (key_pairs / max_tile) >= fill) {
      chosen = v;
      break;
    }
  }
  p.variant = chosen;
  p.R = vars[chosen].R;
  p.NT = vars[chosen].NT;
  const int64_t rpc = static_cast<int64_t>(p.R) * p.NT;
  p.row_blocks = ceil_div(n_rows, rpc);
  p.rows_pad = p.row_blocks * rpc;
  int tile = max_tile;
  while (tile > 16 && p.row_blocks * (key_pairs / tile) < fill) tile /= 2;
  p.tile_pairs = tile;
  const int64_t tiles = key_pairs / tile;
  // Column splits: the grid is row_blocks x splits equal units over `slots` resident CTAs.
  // Take the fewest splits whose last wave is at least 97 % full, else the best one within
  // max(4 waves, 3 splits per row block) units (which bounds the partial buffers).
  const int64_t slots =
      static_cast<int64_t>(sms) *
      occupancy_for(D, grad, chosen, pass_smem_bytes(D, tile, stages_for(D)));
  const int64_t max_units = std::max<int64_t>(4 * slots, 3 * p.row_blocks);
  int64_t best_s = 1;
  double best_eff = -1.0;
  const int64_t s_max = std::min<int64_t>(std::min<int64_t>(tiles, 4096), 65535);
  for (int64_t sp = 1; sp <= s_max; ++sp) {
    const int64_t per = ceil_div(tiles, sp);
    const int64_t s_real = ceil_div(tiles, per);
    if (sp > 1 && p.row_blocks * s_real > max_units) break;
    const double waves = static_cast<double>(p.row_blocks * s_real) / static_cast<double>(slots);
    const double eff = waves / std::ceil(waves);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best_s = s_real;
    }
    if (waves >= 1.0 && eff >= 0.97) break;
  }
  const int64_t per = ceil_div(tiles, best_s);
  p.n_splits = static_cast<int>(ceil_div(tiles, per));
  p.pairs_per_split = per * tile;
  return p;
}

int64_t partial_floats(const Plan& p, int D, bool grad) {
  if (p.n_splits <= 1) return 0;
  return static_cast<int64_t>(p.n_splits) * p.rows_pad * (2 + (grad ? D : 0));
}

// Screens per direction and call that evaluate the anchor tiles (and record each row's best
// anchor key) before the later screens use the recorded keys.
constexpr int kAnchorRecords = 2;

// Queue mode: passes on sorted clouds whose key tiles are whole screening tiles run on the
// unit plan of fs_screen.cuh. The kept-tile masks take one bit per (row block, key tile),
// capped at kMaskCapWords words; larger problems run unscreened in split mode.
constexpr int64_t kMaskCapWords = int64_t(64) << 20;  // 256 MiB
// Unit budget: up to kUnitWaves waves of resident CTAs (many short units balance the SMs),
// but at most kUnitsPerBlock per row block, which keeps the partials' memory in proportion
// to the problem (4 x the rows' own (2 + channels) floats).
constexpr int kUnitWaves = 32;
constexpr int kUnitsPerBlock = 4;

struct QPlan {
  bool on;
  int64_t rb;         // row blocks
  int RB;             // rows per row block
  int mask_words;     // 32-tile mask words per row block
  int64_t budget;     // C = max(1, ceil(kept / budget)) tiles per unit
  int64_t units_max;  // budget + rb bounds the number of units
};

QPlan make_qplan(const Plan& pl, int64_t key_pairs, int D, bool grad, int sms, bool sorted) {
  QPlan q{};
  const int64_t tiles = key_pairs / (kScreenTile / 2);
  q.RB = kQueueShape.R * kQueueShape.NT;
  q.rb = ceil_div(pl.n_rows, q.RB);
  q.mask_words = static_cast<int>(ceil_div(tiles, 32));
  q.on = sorted && D <= 16 && pl.tile_pairs == kScreenTile / 2 && tiles >= 2 &&
         q.rb * q.mask_words <= kMaskCapWords;
  if (!q.on) return q;
  const int64_t slots = static_cast<int64_t>(sms) *
                        occupancy_for(D, grad, kQueueVariant,
                                      pass_smem_bytes(D, kScreenTile / 2, kQueueStages, 0, true),
                                      true);
  q.budget = std::max<int64_t>(1, std::min<int64_t>(kUnitWaves * slots, kUnitsPerBlock * q.rb));
  q.units_max = q.budget + q.rb;
  return q;
}

int64_t queue_partial_floats(const QPlan& q, int D, bool grad) {
  return q.on ? q.units_max * q.RB * (2 + (grad ? D : 0)) : 0;
}

// Points wider than 16 coordinates take the tensor-core passes; the padded width is 32, 48
// or 64, and above 64 a multiple of 64 (the K-chunks of the wide passes).
int tc_dim(int d) {
  if (d <= 16) return 0;
  if (d <= 64) return d <= 32 ? 32 : (d <= 48 ? 48 : 64);
  return static_cast<int>(round_up(d, kTcChunk));
}
inline bool tc_wide(int Dtc) { return Dtc > 64; }
int64_t tc_pad(int64_t count) { return round_up(count, kTcRows); }

struct TcPlan {
  int64_t row_blocks, rows_pad, key_tiles, tiles_per_split;
  int n_splits;
};

int occupancy_tc(int Dtc);  // defined with the launchers

TcPlan make_tc_plan(int64_t n_rows, int64_t n_keys, int Dtc, int sms) {
  TcPlan p{};
  p.row_blocks = ceil_div(n_rows, kTcRows);
  p.rows_pad = p.row_blocks * kTcRows;
  p.key_tiles = tc_pad(n_keys) / kTcCols;
  const int64_t slots = static_cast<int64_t>(sms) * occupancy_tc(Dtc);
  const int64_t max_units = std::max<int64_t>(4 * slots, 3 * p.row_blocks);
  int64_t best_s = 1;
  double best_eff = -1.0;
  const int64_t s_max = std::min<int64_t>(p.key_tiles, 4096);
  for (int64_t sp = 1; sp <= s_max; ++sp) {
    const int64_t per = ceil_div(p.key_tiles, sp);
    const int64_t s_real = ceil_div(p.key_tiles, per);
    if (sp > 1 && p.row_blocks * s_real > max_units) break;
    const double waves = static_cast<double>(p.row_blocks * s_real) / static_cast<double>(slots);
    const double eff = waves / std::ceil(waves);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best_s = s_real;
    }
    if (waves >= 1.0 && eff >= 0.97) break;
  }
  p.tiles_per_split = ceil_div(p.key_tiles, best_s);
  p.n_splits = static_cast<int>(ceil_div(p.key_tiles, p.tiles_per_split));
  return p;
}

constexpr size_t kAlign = 256;
constexpr int kScalarDoubles = 256;  // 2 KiB of float64 scalars

// Offsets (in doubles) inside the scalar block.
constexpr int kSumX = 0;      // [64] coordinate sums of x (tensor-core path)
constexpr int kSumY = 64;     // [64] coordinate sums of y
constexpr int kSumA = 128;
constexpr int kSumB = 129;
constexpr int kAccRow = 130;  // [3]
constexpr int kAccCol = 133;  // [3]
constexpr int kDotFA = 136;
constexpr int kDotGB = 137;
constexpr int kHashX = 138;    // uint64: fingerprint of x's coordinates
constexpr int kHashY = 139;    // uint64: fingerprint of y's coordinates
constexpr int kFlags = 140;   // unsigned, in the bytes of this double
constexpr int kErr = 141;     // unsigned
constexpr int kMaxAbs = 142;  // unsigned: float bits of the largest |coordinate| of x and y
constexpr int kBox = 144;     // ints: ordered lo[3], hi[3] of the first three coordinates
constexpr int kDmin = 147;    // ints: ordered smallest key-bias change of x, of y
constexpr int kEval = 148;    // uint64[3]: pairs evaluated by sorted passes, by TimedKind
constexpr int kQueue = 151;   // ints: tiles per unit C and unit count U of the last queue plan
constexpr int kKept = 152;    // int64: kept tiles K of the last queue plan
constexpr int kPotChange = 153;  // unsigned: float bits of the largest potential change
constexpr int kCgDots = 156;     // [4] float64: the HVP solve's dot products and sums
constexpr int kPayMax = 160;     // unsigned: float bits of the largest |payload| of an apply pass
constexpr int kPayInv = 161;     // float: 1 / s of that pass's payload image
constexpr int kVMax = 162;       // unsigned: float bits of max |v| (HVP difference pass)
constexpr int kVInv = 163;       // float: 1 / s_v of its vector image
constexpr int kDgMax = 164;      // unsigned: float bits of max |dg|
// [kSortMemoWords] uint64 from here: the record of the last sort done in this workspace,
// which prepare() does not clear (everything before it is cleared at every call)
constexpr int kSortMemo = 240;
constexpr unsigned long long kSortMagic = 0x536f72744d656d6full;  // "SortMemo"
static_assert(kSortMemo + kSortMemoWords <= kScalarDoubles, "sort record outside the scalar block");

struct Layout {
  int D;       // padded dimension of the FMA path
  int KP;      // floats per key pair
  int64_t px;  // key pairs of x (padded)
  int64_t py;
  int Dtc;     // padded dimension of the tensor-core path, 0 if unused
  int64_t tx, ty;  // points of x and y padded to whole 128-point tiles (tensor-core path)
  size_t off_scalars, off_kx, off_ky, off_lwx, off_lwy, off_part, total;
  size_t off_img_x, off_img_y, off_nrm_x, off_nrm_y, off_hy_x, off_hy_y;
  // apply passes (d > 16): the rows' LSE2 offsets and plan masses (rows x, then rows y), a
  // payload image; the HVP's difference pass: the rows' vector image, per-row (qs, x'.v),
  // the keys' padded dg
  size_t off_tc_lse, off_tc_mass, off_tc_pay, off_tc_vimg, off_tc_vrow, off_tc_dg;
  // wide layouts (d > 64): per-coordinate sums of both clouds and the centre
  size_t off_tc_sums, off_tc_ctr;
  // spatial order and screening (FMA path): permutations, sort keys, per-tile boxes and bias
  // maxima, and the LSE2 of every row in its last pass
  bool sorted;
  int64_t sort_n;  // keys of the bitonic sort (power of two, >= kSortSmem)
  size_t off_perm_x, off_perm_y, off_code_x, off_code_y, off_sortkeys, off_box_x, off_box_y, off_hmax_x, off_hmax_y,
      off_lse_x, off_lse_y;
  // queue mode: kept-tile masks, kept counts, unit starts and unit -> row block
  size_t off_kmask, off_kcount, off_ustart, off_unit_rb, off_unit_j;
  // screening: each row's recorded anchor key (rows x, rows y); the 16-point group records of
  // each cloud (D <= 3) and the rows' thresholds of the last screen
  size_t off_akey_x, off_akey_y, off_gsum_x, off_gsum_y, off_rowthr;
  // general solve: deferred biases of x (symmetric schedule), potentials at the last check
  size_t off_defer, off_fprev, off_gprev;
  // transport products and the Hessian-vector product (layouts asked with acc_ch > 0):
  // keys with payload channels and the vectors of the HVP's conjugate-gradient solve
  size_t off_paykeys, off_hvp;
  // cosine cost: the normalised copies of x and y
  size_t off_cos;
  int64_t part_floats;
};

constexpr int kTransportChannels = 16;  // payload channels of one transport pass, at most

// Floats of the HVP's vectors, in the order hvp_impl carves them: ft and a spare row vector
// (2n); the solution, residual, direction, product and transport output over n + m (5);
// the gradient, the difference sums and 2v (3 n d); the column pass's payload (n (d + 2))
// and output (m (d + 2)); the column sums (m); the best solution so far (n + m).
inline int64_t hvp_floats(int64_t n, int64_t m, int d) {
  return 2 * n + 6 * (n + m) + 3 * n * d + (n + m) * (d + 2) + m + 64;
}

inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

Layout make_layout(int64_t n, int64_t m, int d, int sms, int acc_ch = 0, bool cosine = false) {
  Layout L{};
  L.D = padded_dim(d);
  L.KP = key_pair_floats(L.D);
  L.px = pairs_pad(n);
  L.py = pairs_pad(m);
  L.Dtc = tc_dim(d);
  L.sorted = L.Dtc == 0;
  int64_t pf = 0, mask_words = 0, rb_max = 0, units_max = 0;
  for (int grad = 0; grad < 2; ++grad) {
    for (int rows_x = 0; rows_x < 2; ++rows_x) {
      const int64_t key_pairs = rows_x ? L.py : L.px;
      const Plan pl = make_plan(rows_x ? n : m, key_pairs, L.D, grad, sms);
      const int ch = std::max(L.D, acc_ch);  // accumulated channels of a gradient-like pass
      pf = std::max(pf, partial_floats(pl, ch, grad));
      const QPlan q = make_qplan(pl, key_pairs, L.D, grad, sms, L.sorted);
      if (q.on) {
        pf = std::max(pf, queue_partial_floats(q, ch, grad));
        mask_words = std::max(mask_words, q.rb * q.mask_words);
        rb_max = std::max(rb_max, q.rb);
        units_max = std::max(units_max, q.units_max);
      }
    }
  }
  L.tx = tc_pad(n);
  L.ty = tc_pad(m);
  if (L.Dtc) {
    // potential passes: (max, sum) per split and row; apply passes: (sum, NC channels and,
    // for the difference pass, a second sum)
    const int64_t nc = tc_wide(L.Dtc) ? kPayChannels : std::max<int64_t>(L.Dtc, kPayChannels);
    for (const TcPlan& tp : {make_tc_plan(n, m, L.Dtc, sms), make_tc_plan(m, n, L.Dtc, sms)})
      if (tp.n_splits > 1) pf = std::max<int64_t>(pf, (2 + nc) * tp.n_splits * tp.rows_pad);
  }
  L.part_floats = pf;
  size_t o = 0;
  L.off_scalars = o;
  o = align_up(o + kScalarDoubles * sizeof(double));
  L.off_kx = o;
  o = align_up(o + static_cast<size_t>(L.px) * L.KP * sizeof(float));
  L.off_ky = o;
  o = align_up(o + static_cast<size_t>(L.py) * L.KP * sizeof(float));
  L.off_lwx = o;
  o = align_up(o + static_cast<size_t>(2 * L.px) * sizeof(float));
  L.off_lwy = o;
  o = align_up(o + static_cast<size_t>(2 * L.py) * sizeof(float));
  L.off_part = o;
  o = align_up(o + static_cast<size_t>(pf) * sizeof(float));
  if (L.Dtc) {
    const size_t kbytes = static_cast<size_t>(2 * L.Dtc) * 2;  // [hi | lo] fp16 per point
    L.off_img_x = o;
    o = align_up(o + static_cast<size_t>(L.tx) * kbytes);
    L.off_img_y = o;
    o = align_up(o + static_cast<size_t>(L.ty) * kbytes);
    L.off_nrm_x = o;
    o = align_up(o + static_cast<size_t>(L.tx) * sizeof(float));
    L.off_nrm_y = o;
    o = align_up(o + static_cast<size_t>(L.ty) * sizeof(float));
    L.off_hy_x = o;
    o = align_up(o + static_cast<size_t>(L.tx) * sizeof(float));
    L.off_hy_y = o;
    o = align_up(o + static_cast<size_t>(L.ty) * sizeof(float));
    if (tc_wide(L.Dtc)) {
      L.off_tc_sums = o;
      o = align_up(o + static_cast<size_t>(2 * L.Dtc) * sizeof(double));
      L.off_tc_ctr = o;
      o = align_up(o + static_cast<size_t>(L.Dtc) * sizeof(double));
    }
    const int64_t tmax = std::max(L.tx, L.ty);
    L.off_tc_lse = o;
    o = align_up(o + static_cast<size_t>(2 * tmax) * sizeof(float));
    L.off_tc_mass = o;
    o = align_up(o + static_cast<size_t>(2 * tmax) * sizeof(float));
    if (acc_ch > 0 || tc_wide(L.Dtc)) {
      // the payload image: transport products, and the gradient of wide points (P y)
      L.off_tc_pay = o;
      o = align_up(o + static_cast<size_t>(tmax) * 2 * kPayChannels * 2);
    }
    if (acc_ch > 0) {
      L.off_tc_vimg = o;
      o = align_up(o + static_cast<size_t>(L.tx) * 2 * L.Dtc * 2);
      L.off_tc_vrow = o;
      o = align_up(o + static_cast<size_t>(2 * L.tx) * sizeof(float));
      L.off_tc_dg = o;
      o = align_up(o + static_cast<size_t>(tmax) * sizeof(float));
    }
  }
  if (L.sorted) {
    int64_t sn = kSortSmem;
    while (sn < std::max(n, m)) sn <<= 1;
    L.sort_n = sn;
    const int64_t tiles_x = L.px / kPairPad, tiles_y = L.py / kPairPad;
    L.off_perm_x = o;
    o = align_up(o + static_cast<size_t>(n) * sizeof(int));
    L.off_perm_y = o;
    o = align_up(o + static_cast<size_t>(m) * sizeof(int));
    L.off_code_x = o;
    o = align_up(o + static_cast<size_t>(n) * sizeof(unsigned));
    L.off_code_y = o;
    o = align_up(o + static_cast<size_t>(m) * sizeof(unsigned));
    L.off_sortkeys = o;
    o = align_up(o + static_cast<size_t>(sn) * sizeof(uint64_t));
    // tile summaries followed by their super-tile summaries
    const int64_t sx = tiles_x + ceil_div(tiles_x, kSuper), sy = tiles_y + ceil_div(tiles_y, kSuper);
    L.off_box_x = o;
    o = align_up(o + static_cast<size_t>(sx) * 2 * L.D * sizeof(float));
    L.off_box_y = o;
    o = align_up(o + static_cast<size_t>(sy) * 2 * L.D * sizeof(float));
    L.off_hmax_x = o;
    o = align_up(o + static_cast<size_t>(sx) * sizeof(float));
    L.off_hmax_y = o;
    o = align_up(o + static_cast<size_t>(sy) * sizeof(float));
    L.off_lse_x = o;
    o = align_up(o + static_cast<size_t>(n) * sizeof(float));
    L.off_lse_y = o;
    o = align_up(o + static_cast<size_t>(m) * sizeof(float));
    if (L.D <= 3) {
      L.off_gsum_x = o;
      o = align_up(o + static_cast<size_t>(tiles_x) * kTileGroupFloats * sizeof(float));
      L.off_gsum_y = o;
      o = align_up(o + static_cast<size_t>(tiles_y) * kTileGroupFloats * sizeof(float));
      L.off_rowthr = o;
      o = align_up(o + static_cast<size_t>(std::max(n, m)) * sizeof(float));
    }
    L.off_akey_x = o;
    o = align_up(o + static_cast<size_t>(n) * sizeof(int));
    L.off_akey_y = o;
    o = align_up(o + static_cast<size_t>(m) * sizeof(int));
    L.off_kmask = o;
    o = align_up(o + static_cast<size_t>(mask_words) * sizeof(unsigned));
    L.off_kcount = o;
    o = align_up(o + static_cast<size_t>(rb_max) * sizeof(int));
    L.off_ustart = o;
    o = align_up(o + static_cast<size_t>(rb_max + 1) * sizeof(int));
    L.off_unit_rb = o;
    o = align_up(o + static_cast<size_t>(units_max) * sizeof(int));
    L.off_unit_j = o;
    o = align_up(o + static_cast<size_t>(units_max) * sizeof(int));
  }
  L.off_defer = o;
  o = align_up(o + static_cast<size_t>(std::max(n, L.tx)) * sizeof(float));
  L.off_fprev = o;
  o = align_up(o + static_cast<size_t>(n) * sizeof(float));
  L.off_gprev = o;
  o = align_up(o + static_cast<size_t>(m) * sizeof(float));
  if (acc_ch > 0) {
    if (!L.Dtc) {  // payload keys of the FMA transport passes
      L.off_paykeys = o;
      o = align_up(o + static_cast<size_t>(std::max(L.px, L.py)) * pair_floats(L.D, acc_ch) *
                           sizeof(float));
    }
    L.off_hvp = o;
    o = align_up(o + static_cast<size_t>(hvp_floats(n, m, d)) * sizeof(float));
  }
  if (cosine) {
    L.off_cos = o;
    o = align_up(o + static_cast<size_t>(n + m) * d * sizeof(float));
  }
  L.total = o;
  return L;
}

bool shape_ok(const fs_problem* p) {
  return p && p->n >= 1 && p->m >= 1 && p->d >= 1 && p->n <= (int64_t(1) << 40) &&
         p->m <= (int64_t(1) << 40);
}

inline bool aligned4(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; }

// ---------------- kernel dispatch ----------------

template <int D, int R, int NT, int MODE, int NP, int G, int MINB, int ST = kStages>
struct PassKernel {
  // unscreened launches; screened ones (fnq) skip 16-point groups when D <= 3
  static constexpr bool kGroups = D <= 3 && NT == 32;
  static constexpr auto fn = lse_pass_kernel<D, R, NT, G, MODE, NP, MINB, ST, false>;
  static constexpr auto fnq = lse_pass_kernel<D, R, NT, G, MODE, NP, MINB, ST, kGroups>;
  static void set_smem_attr() {
    static bool done = false;  // idempotent, so a race between threads is harmless
    if (!done) {
      CK(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(pass_smem_bytes(D, 128, ST, NP))));
      CK(cudaFuncSetAttribute(fnq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(pass_smem_bytes(D, 128, ST, NP, kGroups))));
      done = true;
    }
  }
  static void launch(const PassParams& P0, const Plan& pl, cudaStream_t st) {
    set_smem_attr();
    PassParams P = P0;
    P.group_recs = 0;  // unscreened: stages hold key tiles only
    dim3 grid(static_cast<unsigned>(pl.row_blocks), static_cast<unsigned>(pl.n_splits));
    fn<<<grid, NT, pass_smem_bytes(D, pl.tile_pairs, ST, NP), st>>>(P);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  static void launch_queue(const PassParams& P0, int64_t units, cudaStream_t st) {
    set_smem_attr();
    PassParams P = P0;
    P.group_recs = kGroups && P.row_thr && P.gsum ? 1 : 0;
    fnq<<<static_cast<unsigned>(units), NT,
          pass_smem_bytes(D, kScreenTile / 2, ST, NP, P.group_recs != 0), st>>>(P);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  static void screen(const PassParams& P, int64_t rb, unsigned* kmask, int* kcount,
                     cudaStream_t st) {
    if constexpr (D <= 16 && NT == 32) {  // one warp per row block, FMA-path widths only
      const size_t smem = P.key_supers <= kSupCache ? P.key_supers * sizeof(float) : 0;
      screen_kernel<D, R><<<static_cast<unsigned>(rb), 32, smem, st>>>(P, kmask, kcount);
      CK(cudaGetLastError());
      g_launches.fetch_add(1, std::memory_order_relaxed);
    }
  }
  static int occupancy(size_t smem, bool queue) {
    int n = 0;
    set_smem_attr();
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, queue ? fnq : fn, NT, smem) !=
            cudaSuccess ||
        n < 1) {
      cudaGetLastError();
      n = MINB;
    }
    return n;
  }
};

// The kernel of (D, pass type, variant): calls op.template run<Kernel>().
template <int D, typename Op>
void with_pass_kernel(int sel, int variant, Op&& op) {
  (void)variant;
  if constexpr (D > 16) {  // the gradient of wide points; potentials run on the tensor cores
    if (sel == kSelGrad)
      op.template run<PassKernel<D, 1, 128, kModeGrad, 0, 4, 1>>();
    else
      op.template run<PassKernel<D, 1, 128, kModeLse, 0, 4, 1>>();
  } else {
    constexpr int S = kNarrowStages;
    switch (sel) {
      case kSelGrad: op.template run<PassKernel<D, 2, 32, kModeGrad, 0, 8, 16, S>>(); break;
      case kSelPay1: op.template run<PassKernel<D, 2, 32, kModePay, 1, 8, 20, S>>(); break;
      case kSelPay4: op.template run<PassKernel<D, 2, 32, kModePay, 4, 8, 16, S>>(); break;
      case kSelPay16: op.template run<PassKernel<D, 2, 32, kModePay, 16, 8, 8, S>>(); break;
      case kSelDiff: op.template run<PassKernel<D, 2, 32, kModeDiff, 1, 8, 8, S>>(); break;
      default: op.template run<PassKernel<D, 2, 32, kModeLse, 0, 8, 24, S>>(); break;
    }
  }
}

struct LaunchOp {
  const PassParams& P;
  const Plan& pl;
  cudaStream_t st;
  template <typename K>
  void run() { K::launch(P, pl, st); }
};

struct QueueOp {
  const PassParams& P;
  int64_t units;
  cudaStream_t st;
  template <typename K>
  void run() { K::launch_queue(P, units, st); }
};

struct ScreenOp {
  const PassParams& P;
  int64_t rb;
  unsigned* kmask;
  int* kcount;
  cudaStream_t st;
  template <typename K>
  void run() { K::screen(P, rb, kmask, kcount, st); }
};

struct OccupancyOp {
  size_t smem;
  bool queue;
  int result = 1;
  template <typename K>
  void run() { result = K::occupancy(smem, queue); }
};

template <int D>
void launch_pass_d(const PassParams& P, const Plan& pl, int sel, cudaStream_t st) {
  with_pass_kernel<D>(sel, pl.variant, LaunchOp{P, pl, st});
}

template <int D>
void launch_queue_d(const PassParams& P, int64_t units, int sel, cudaStream_t st) {
  with_pass_kernel<D>(sel, kQueueVariant, QueueOp{P, units, st});
}

template <int D>
void launch_screen_d(const PassParams& P, int64_t rb, unsigned* kmask, int* kcount,
                     cudaStream_t st) {
  with_pass_kernel<D>(kSelLse, kQueueVariant, ScreenOp{P, rb, kmask, kcount, st});
}

template <int D>
void occupancy_d(bool grad, int variant, OccupancyOp* op) {
  with_pass_kernel<D>(grad ? kSelGrad : kSelLse, variant, *op);
}

template <int D>
void launch_combine_d(const PassParams& P, int sel, cudaStream_t st) {
  const unsigned blocks = static_cast<unsigned>(ceil_div(P.n_rows, 256));
  switch (sel) {
    case kSelGrad: combine_kernel<D, kModeGrad, D><<<blocks, 256, 0, st>>>(P); break;
    case kSelPay1: combine_kernel<D, kModePay, 1><<<blocks, 256, 0, st>>>(P); break;
    case kSelPay4: combine_kernel<D, kModePay, 4><<<blocks, 256, 0, st>>>(P); break;
    case kSelPay16: combine_kernel<D, kModePay, 16><<<blocks, 256, 0, st>>>(P); break;
    case kSelDiff: combine_kernel<D, kModeDiff, D><<<blocks, 256, 0, st>>>(P); break;
    default: combine_kernel<D, kModeLse, 1><<<blocks, 256, 0, st>>>(P); break;
  }
  CK(cudaGetLastError());
  g_launches.fetch_add(1, std::memory_order_relaxed);
}

#define FS_DISPATCH_D(D, FN, ...)                 \
  switch (D) {                                    \
    case 1: FN<1>(__VA_ARGS__); break;            \
    case 2: FN<2>(__VA_ARGS__); break;            \
    case 3: FN<3>(__VA_ARGS__); break;            \
    case 4: FN<4>(__VA_ARGS__); break;            \
    case 8: FN<8>(__VA_ARGS__); break;            \
    case 16: FN<16>(__VA_ARGS__); break;          \
    case 32: FN<32>(__VA_ARGS__); break;          \
    default: FN<64>(__VA_ARGS__); break;          \
  }

template <int Dtc>
struct TcKernel {
  static constexpr auto fn = lse_pass_tc_kernel<Dtc>;
  static void set_smem_attr() {
    static bool done = false;  // idempotent, so a race between threads is harmless
    if (!done) {
      CK(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(TcShape<Dtc>::SMEM)));
      done = true;
    }
  }
  static void launch(const PassParams& P, const TcParams& T, const TcPlan& pl, cudaStream_t st) {
    set_smem_attr();
    dim3 grid(static_cast<unsigned>(pl.row_blocks), static_cast<unsigned>(pl.n_splits));
    fn<<<grid, kTcThreads, TcShape<Dtc>::SMEM, st>>>(P, T);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  static int occupancy() {
    int n = 0;
    try {
      set_smem_attr();
    } catch (const CudaFail&) {
      cudaGetLastError();
      return 1;
    }
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kTcThreads, TcShape<Dtc>::SMEM) !=
            cudaSuccess ||
        n < 1) {
      cudaGetLastError();
      n = 1;
    }
    return n;
  }
};

// Resident CTAs per SM of the potential pass: shared memory's limit, and TMEM's (each CTA
// allocates kTcTmemCols of the SM's 512 columns; a CTA beyond that would wait in its
// allocation).
int occupancy_tc(int Dtc) {
  int n = 1;
  if (tc_wide(Dtc)) return 1;  // one 194 KB CTA per SM
  switch (Dtc) {
    case 32: n = TcKernel<32>::occupancy(); break;
    case 48: n = TcKernel<48>::occupancy(); break;
    default: n = TcKernel<64>::occupancy(); break;
  }
  return std::max(1, std::min(n, static_cast<int>(512u / kTcTmemCols)));
}

void launch_tc_wide(const PassParams& P, const TcParams& T, const TcPlan& pl, cudaStream_t st) {
  static bool done = false;  // idempotent, so a race between threads is harmless
  if (!done) {
    CK(cudaFuncSetAttribute(lse_pass_tcw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            static_cast<int>(TcWideShape::SMEM)));
    done = true;
  }
  dim3 grid(static_cast<unsigned>(pl.row_blocks), static_cast<unsigned>(pl.n_splits));
  lse_pass_tcw_kernel<<<grid, kTcThreads, TcWideShape::SMEM, st>>>(P, T);
  CK(cudaGetLastError());
  g_launches.fetch_add(1, std::memory_order_relaxed);
}

void launch_tc(int Dtc, const PassParams& P, const TcParams& T, const TcPlan& pl, cudaStream_t st) {
  if (tc_wide(Dtc)) {
    launch_tc_wide(P, T, pl, st);
    return;
  }
  switch (Dtc) {
    case 32: TcKernel<32>::launch(P, T, pl, st); break;
    case 48: TcKernel<48>::launch(P, T, pl, st); break;
    default: TcKernel<64>::launch(P, T, pl, st); break;
  }
}

template <int Dtc, int NC, int MODE>
struct TcApplyKernel {
  static constexpr auto fn = lse_apply_tc_kernel<Dtc, NC, MODE>;
  static constexpr size_t SMEM = TcApplyShape<Dtc, NC, MODE>::SMEM;
  static void launch(const PassParams& P, const TcParams& T, const TcApply& A, const TcPlan& pl,
                     cudaStream_t st) {
    static bool done = false;  // idempotent, so a race between threads is harmless
    if (!done) {
      CK(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(SMEM)));
      done = true;
    }
    dim3 grid(static_cast<unsigned>(pl.row_blocks), static_cast<unsigned>(pl.n_splits));
    fn<<<grid, kTcThreads, SMEM, st>>>(P, T, A);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (pl.n_splits > 1) {
      tc_apply_combine_kernel<NC, MODE><<<static_cast<unsigned>(ceil_div(P.n_rows, 256)), 256, 0,
                                          st>>>(P, A);
      CK(cudaGetLastError());
      g_launches.fetch_add(1, std::memory_order_relaxed);
    }
  }
};

void launch_apply_tc(int Dtc, int mode, const PassParams& P, const TcParams& T, const TcApply& A,
                     const TcPlan& pl, cudaStream_t st) {
  if (tc_wide(Dtc)) {  // transport products only (the gradient runs as one)
    static bool done = false;
    if (!done) {
      CK(cudaFuncSetAttribute(lse_apply_tcw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(TcWideShape::APPLY_SMEM)));
      done = true;
    }
    dim3 grid(static_cast<unsigned>(pl.row_blocks), static_cast<unsigned>(pl.n_splits));
    lse_apply_tcw_kernel<<<grid, kTcThreads, TcWideShape::APPLY_SMEM, st>>>(P, T, A);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (pl.n_splits > 1) {
      tc_apply_combine_kernel<kPayChannels, kApplyPay>
          <<<static_cast<unsigned>(ceil_div(P.n_rows, 256)), 256, 0, st>>>(P, A);
      CK(cudaGetLastError());
      g_launches.fetch_add(1, std::memory_order_relaxed);
    }
    return;
  }
  if (mode == kApplyGrad) {
    switch (Dtc) {
      case 32: TcApplyKernel<32, 32, kApplyGrad>::launch(P, T, A, pl, st); break;
      case 48: TcApplyKernel<48, 48, kApplyGrad>::launch(P, T, A, pl, st); break;
      default: TcApplyKernel<64, 64, kApplyGrad>::launch(P, T, A, pl, st); break;
    }
  } else if (mode == kApplyPay) {
    switch (Dtc) {
      case 32: TcApplyKernel<32, kPayChannels, kApplyPay>::launch(P, T, A, pl, st); break;
      case 48: TcApplyKernel<48, kPayChannels, kApplyPay>::launch(P, T, A, pl, st); break;
      default: TcApplyKernel<64, kPayChannels, kApplyPay>::launch(P, T, A, pl, st); break;
    }
  } else {
    switch (Dtc) {
      case 32: TcApplyKernel<32, 32, kApplyDiff>::launch(P, T, A, pl, st); break;
      case 48: TcApplyKernel<48, 48, kApplyDiff>::launch(P, T, A, pl, st); break;
      default: TcApplyKernel<64, 64, kApplyDiff>::launch(P, T, A, pl, st); break;
    }
  }
}

template <int Dtc>
void launch_image(const float* pts, int64_t count, int d, const TcCenter& ctr, float scale,
                  unsigned char* img, float* nrm, int64_t pad, cudaStream_t st) {
  build_image_kernel<Dtc><<<static_cast<unsigned>(ceil_div(pad, 256)), 256, 0, st>>>(
      pts, count, d, ctr, scale, img, nrm, pad);
  CK(cudaGetLastError());
  g_launches.fetch_add(1, std::memory_order_relaxed);
}

int occupancy_for(int D, bool grad, int variant, size_t smem, bool queue) {
  OccupancyOp op{smem, queue};
  try {
    FS_DISPATCH_D(D, occupancy_d, grad, variant, &op);
  } catch (const CudaFail&) {
    cudaGetLastError();
    op.result = 1;
  }
  return op.result;
}

template <int D>
void launch_pack_d(const float* pts, int64_t count, int d, const float* w, float wu,
                   const int* perm, float* keys, float* lw, int64_t pp, cudaStream_t st) {
  const unsigned blocks = static_cast<unsigned>(ceil_div(2 * pp, 256));
  pack_kernel<D><<<blocks, 256, 0, st>>>(pts, count, d, w, wu, perm, keys, lw, pp);
  CK(cudaGetLastError());
  g_launches.fetch_add(1, std::memory_order_relaxed);
}

template <int D>
void launch_payload_keys_d(const float* keys, int64_t count, int64_t pairs, const float* pay, int k,
                           int stride, const int* perm, float* out, int np, cudaStream_t st) {
  const unsigned blocks = static_cast<unsigned>(ceil_div(2 * pairs, 256));
  if constexpr (D <= 16) {
    if (np == 1)
      payload_keys_kernel<D, 1><<<blocks, 256, 0, st>>>(keys, count, pairs, pay, k, stride, perm, out);
    else if (np == 4)
      payload_keys_kernel<D, 4><<<blocks, 256, 0, st>>>(keys, count, pairs, pay, k, stride, perm, out);
    else
      payload_keys_kernel<D, 16><<<blocks, 256, 0, st>>>(keys, count, pairs, pay, k, stride, perm, out);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
}

template <int D>
void launch_cells_d(const float* keys, int64_t count, int32_t d, const float* w, float wu,
                    const int* perm, int cell_points, float* pts, float* mass, int64_t cells,
                    cudaStream_t st) {
  if constexpr (D <= 16) {
    cell_kernel<D><<<static_cast<unsigned>(cells), 256, 0, st>>>(keys, count, d, w, wu, perm,
                                                                 cell_points, pts, mass);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
}

template <int D>
void launch_apply_bias_d(float* keys, const float* defer_h, int64_t count, int* dmin,
                         cudaStream_t st) {
  apply_bias_kernel<D><<<static_cast<unsigned>(ceil_div(count, 256)), 256, 0, st>>>(keys, defer_h,
                                                                                    count, dmin);
  CK(cudaGetLastError());
  g_launches.fetch_add(1, std::memory_order_relaxed);
}

template <int D>
void launch_bias_d(float* keys, int64_t count, const float* pot, const int* perm, const float* lw,
                   double kappa, cudaStream_t st) {
  const unsigned blocks = static_cast<unsigned>(ceil_div(count, 256));
  key_bias_kernel<D><<<blocks, 256, 0, st>>>(keys, count, pot, perm, lw, kappa);
  CK(cudaGetLastError());
  g_launches.fetch_add(1, std::memory_order_relaxed);
}

template <int D>
void launch_tile_box_d(const float* keys, int64_t count, int64_t tiles, float* box, float* gsum,
                       cudaStream_t st) {
  // tile boxes, then super-tile boxes behind them (lower corners by min, upper by max)
  tile_box_kernel<D><<<static_cast<unsigned>(tiles), 256, 0, st>>>(keys, count, box, tiles, gsum);
  CK(cudaGetLastError());
  const int64_t supers = ceil_div(tiles, kSuper);
  super_reduce_kernel<<<static_cast<unsigned>(ceil_div(supers, 256)), 256, 0, st>>>(
      box, tiles, box + 2 * D * tiles, supers, 2 * D, D);
  CK(cudaGetLastError());
  g_launches.fetch_add(2, std::memory_order_relaxed);
}

template <int D>
void launch_tile_hmax_d(const float* keys, int64_t count, int64_t tiles, float* hmax, float* gsum,
                        cudaStream_t st) {
  tile_hmax_kernel<D><<<static_cast<unsigned>(tiles), 256, 0, st>>>(keys, count, hmax, gsum);
  CK(cudaGetLastError());
  const int64_t supers = ceil_div(tiles, kSuper);
  super_reduce_kernel<<<static_cast<unsigned>(ceil_div(supers, 256)), 256, 0, st>>>(
      hmax, tiles, hmax + tiles, supers, 1, 0);
  CK(cudaGetLastError());
  g_launches.fetch_add(2, std::memory_order_relaxed);
}

// Morton order of one cloud: keys (code << 32 | index), bitonic sort, permutation.
void sort_cloud(const float* pts, int64_t count, int d, const MortonFrame& F, uint64_t* keys,
                int64_t sort_n, int* perm, unsigned* codes, cudaStream_t st) {
  morton_keys_kernel<<<static_cast<unsigned>(ceil_div(sort_n, 256)), 256, 0, st>>>(
      pts, count, d, F, keys, sort_n);
  CK(cudaGetLastError());
  g_launches.fetch_add(1, std::memory_order_relaxed);
  const unsigned sblocks = static_cast<unsigned>(sort_n / kSortSmem);
  bitonic_smem_kernel<<<sblocks, kSortBlock, 0, st>>>(keys, 0);
  CK(cudaGetLastError());
  g_launches.fetch_add(1, std::memory_order_relaxed);
  for (int64_t k = 2 * kSortSmem; k <= sort_n; k <<= 1) {
    for (int64_t j = k / 2; j >= kSortSmem; j >>= 1) {
      bitonic_global_kernel<<<static_cast<unsigned>(ceil_div(sort_n / 2, 256)), 256, 0, st>>>(
          keys, sort_n, k, j);
      CK(cudaGetLastError());
      g_launches.fetch_add(1, std::memory_order_relaxed);
    }
    bitonic_smem_kernel<<<sblocks, kSortBlock, 0, st>>>(keys, k);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  perm_from_keys_kernel<<<static_cast<unsigned>(ceil_div(count, 256)), 256, 0, st>>>(keys, count,
                                                                                      perm, codes);
  CK(cudaGetLastError());
  g_launches.fetch_add(1, std::memory_order_relaxed);
}

// ---------------- one call's context ----------------

struct Ctx {
  const fs_problem* p;
  cudaStream_t st;
  Layout L;
  int sms;
  unsigned char* ws;
  double* scal;
  float* kx;
  float* ky;
  float* lwx;
  float* lwy;
  float* part;
  double ma, mb;  // weight sums
  double kappa;
  Timer* timer;
  bool use_tc;    // potential and marginal passes on the tensor cores
  unsigned char *img_x, *img_y;
  float *nrm_x, *nrm_y, *hy_x, *hy_y;
  float *tc_lse, *tc_mass;      // apply passes: the rows' LSE2 offsets and plan masses
                                // ([0, tmax): rows x; [tmax, 2 tmax): rows y)
  unsigned char* tc_pay;        // apply passes: payload image
  unsigned char* tc_vimg;       // difference pass: the rows' vector image
  float *tc_vrow, *tc_dg;       // difference pass: per-row (qs, x'.v); the keys' padded dg
  double tc_rkey;               // a bound on |y'_j| and |x'_i| (centred points)
  double* tc_sums;              // wide layouts: coordinate sums of x then y (2 Dtc doubles)
  double* tc_ctr_dev;           // wide layouts: the centre (Dtc doubles)
  std::vector<double> tc_ctr_host;
  bool tc_reuse;                // apply passes keep the offsets of their first pre-pass
  bool tc_valid[2];             // ... per direction (rows x, rows y)
  float c2;       // 2 kappa / s^2
  float tc_scale;  // s: the images' power-of-two scale
  TcCenter tc_ctr;  // the centre the images were built about
  int *perm_x, *perm_y;         // sorted slot -> original index (NULL when unsorted)
  unsigned *code_x, *code_y;    // Morton codes in sorted order (NULL when unsorted)
  uint64_t* sortkeys;
  float *box_x, *box_y, *hmax_x, *hmax_y, *lse_x, *lse_y;
  unsigned* kmask;
  int *kcount, *ustart, *unit_rb, *unit_j;
  int *akey_x, *akey_y;  // screening: each row's recorded anchor key
  float *gsum_x, *gsum_y;  // 16-point group records (D <= 3), or NULL
  float* rowthr;           // the rows' thresholds of the last screen (D <= 3), or NULL
  int anchor_records[2];  // screens that recorded anchor keys in this call (rows x, rows y)
  float *defer, *fprev, *gprev;
  float* paykeys; // transport passes: keys with payload channels
  float* hvp;     // the HVP's vectors
  float ctr[3];   // centre of the clouds' box (first three coordinates)
  fs_problem pn;  // cosine cost: the problem on the normalised copies (c.p points here)
  float *cos_x, *cos_y;
  float alpha;    // symmetric schedule: blend weight of the potential passes (0: plain)
  bool defer_x;   // the next x-row potential pass leaves its biases in `defer`
  bool no_screen;  // screening found to keep most tiles: the rest of the call runs unscreened
  bool screen_on;  // fs_screening_enable's setting, read once at the start of the call
};

// Whether the passes of this call may still screen: sorted clouds, screening enabled when the
// call began, and not switched off by the probe after the first iteration.
inline bool screening_live(const Ctx& c) { return c.L.sorted && c.screen_on && !c.no_screen; }

fs_status check_common(const fs_problem* p, void* ws, size_t ws_bytes, size_t* need_out,
                       int sms, int acc_ch = 0) {
  if (!p) return FS_ERR_NULL;
  if (!shape_ok(p)) return FS_ERR_SHAPE;
  if (p->d > FS_MAX_D) return FS_ERR_UNSUPPORTED_D;
  if (!(std::isfinite(p->eps) && p->eps > 0.0f)) return FS_ERR_EPS;
  if (p->cost != FS_COST_SQEUCLIDEAN && p->cost != FS_COST_COSINE) return FS_ERR_OPTION;
  if (!p->x || !p->y) return FS_ERR_NULL;
  if (!aligned4(p->x) || !aligned4(p->y) || !aligned4(p->a) || !aligned4(p->b))
    return FS_ERR_ALIGNMENT;
  const Layout L = make_layout(p->n, p->m, p->d, sms, acc_ch, p->cost == FS_COST_COSINE);
  *need_out = L.total;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 || ws_bytes < L.total)
    return FS_ERR_WORKSPACE;
  return FS_OK;
}

void carve(Ctx& c, void* ws) {
  c.ws = static_cast<unsigned char*>(ws);
  c.scal = reinterpret_cast<double*>(c.ws + c.L.off_scalars);
  c.kx = reinterpret_cast<float*>(c.ws + c.L.off_kx);
  c.ky = reinterpret_cast<float*>(c.ws + c.L.off_ky);
  c.lwx = reinterpret_cast<float*>(c.ws + c.L.off_lwx);
  c.lwy = reinterpret_cast<float*>(c.ws + c.L.off_lwy);
  c.part = reinterpret_cast<float*>(c.ws + c.L.off_part);
  c.defer = reinterpret_cast<float*>(c.ws + c.L.off_defer);
  c.fprev = reinterpret_cast<float*>(c.ws + c.L.off_fprev);
  c.gprev = reinterpret_cast<float*>(c.ws + c.L.off_gprev);
  if (c.L.off_cos) {
    c.cos_x = reinterpret_cast<float*>(c.ws + c.L.off_cos);
    c.cos_y = c.cos_x + c.p->n * c.p->d;
  }
  if (c.L.off_paykeys) c.paykeys = reinterpret_cast<float*>(c.ws + c.L.off_paykeys);
  if (c.L.off_hvp) c.hvp = reinterpret_cast<float*>(c.ws + c.L.off_hvp);
  if (c.L.Dtc) {
    c.img_x = c.ws + c.L.off_img_x;
    c.img_y = c.ws + c.L.off_img_y;
    c.tc_lse = reinterpret_cast<float*>(c.ws + c.L.off_tc_lse);
    if (c.L.off_tc_sums) {
      c.tc_sums = reinterpret_cast<double*>(c.ws + c.L.off_tc_sums);
      c.tc_ctr_dev = reinterpret_cast<double*>(c.ws + c.L.off_tc_ctr);
    }
    c.tc_mass = reinterpret_cast<float*>(c.ws + c.L.off_tc_mass);
    if (c.L.off_tc_pay) c.tc_pay = c.ws + c.L.off_tc_pay;
    if (c.L.off_tc_vimg) {
      c.tc_vimg = c.ws + c.L.off_tc_vimg;
      c.tc_vrow = reinterpret_cast<float*>(c.ws + c.L.off_tc_vrow);
      c.tc_dg = reinterpret_cast<float*>(c.ws + c.L.off_tc_dg);
    }
    c.nrm_x = reinterpret_cast<float*>(c.ws + c.L.off_nrm_x);
    c.nrm_y = reinterpret_cast<float*>(c.ws + c.L.off_nrm_y);
    c.hy_x = reinterpret_cast<float*>(c.ws + c.L.off_hy_x);
    c.hy_y = reinterpret_cast<float*>(c.ws + c.L.off_hy_y);
  }
  if (c.L.sorted) {
    c.perm_x = reinterpret_cast<int*>(c.ws + c.L.off_perm_x);
    c.perm_y = reinterpret_cast<int*>(c.ws + c.L.off_perm_y);
    c.code_x = reinterpret_cast<unsigned*>(c.ws + c.L.off_code_x);
    c.code_y = reinterpret_cast<unsigned*>(c.ws + c.L.off_code_y);
    c.sortkeys = reinterpret_cast<uint64_t*>(c.ws + c.L.off_sortkeys);
    c.box_x = reinterpret_cast<float*>(c.ws + c.L.off_box_x);
    c.box_y = reinterpret_cast<float*>(c.ws + c.L.off_box_y);
    c.hmax_x = reinterpret_cast<float*>(c.ws + c.L.off_hmax_x);
    c.hmax_y = reinterpret_cast<float*>(c.ws + c.L.off_hmax_y);
    c.lse_x = reinterpret_cast<float*>(c.ws + c.L.off_lse_x);
    c.lse_y = reinterpret_cast<float*>(c.ws + c.L.off_lse_y);
    c.kmask = reinterpret_cast<unsigned*>(c.ws + c.L.off_kmask);
    c.akey_x = reinterpret_cast<int*>(c.ws + c.L.off_akey_x);
    if (c.L.off_gsum_x) {
      c.gsum_x = reinterpret_cast<float*>(c.ws + c.L.off_gsum_x);
      c.gsum_y = reinterpret_cast<float*>(c.ws + c.L.off_gsum_y);
      c.rowthr = reinterpret_cast<float*>(c.ws + c.L.off_rowthr);
    }
    c.akey_y = reinterpret_cast<int*>(c.ws + c.L.off_akey_y);
    c.kcount = reinterpret_cast<int*>(c.ws + c.L.off_kcount);
    c.ustart = reinterpret_cast<int*>(c.ws + c.L.off_ustart);
    c.unit_rb = reinterpret_cast<int*>(c.ws + c.L.off_unit_rb);
    c.unit_j = reinterpret_cast<int*>(c.ws + c.L.off_unit_j);
  }
}

unsigned* flags_ptr(double* scal) { return reinterpret_cast<unsigned*>(scal + kFlags); }
unsigned* err_ptr(double* scal) { return reinterpret_cast<unsigned*>(scal + kErr); }

unsigned reduce_blocks(int64_t count, int sms) {
  return static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(ceil_div(count, 256), sms * 4)));
}

// Validates inputs on the device (one stream sync), packs both clouds and their log-weights.
// `pots` lists potentials to check for finiteness (device pointers with their lengths).
fs_status prepare(Ctx& c, const std::vector<std::pair<const float*, int64_t>>& pots,
                  bool need_tc) {
  if (c.p->cost == FS_COST_COSINE) {
    // every pass below runs on the normalised copies, under the squared-Euclidean cost
    const fs_problem* p0 = c.p;
    normalize_kernel<<<static_cast<unsigned>(ceil_div(p0->n, 256)), 256, 0, c.st>>>(
        p0->x, p0->n, p0->d, c.cos_x);
    CK(cudaGetLastError());
    normalize_kernel<<<static_cast<unsigned>(ceil_div(p0->m, 256)), 256, 0, c.st>>>(
        p0->y, p0->m, p0->d, c.cos_y);
    CK(cudaGetLastError());
    g_launches.fetch_add(2, std::memory_order_relaxed);
    c.pn = *p0;
    c.pn.x = c.cos_x;
    c.pn.y = c.cos_y;
    c.pn.cost = FS_COST_SQEUCLIDEAN;
    c.p = &c.pn;
  }
  const fs_problem* p = c.p;
  c.use_tc = need_tc && c.L.Dtc > 0;
  CK(cudaMemsetAsync(c.scal, 0, kSortMemo * sizeof(double), c.st));
  const int sdims = std::min(p->d, kSortDims);
  if (c.L.sorted) {
    // bounding box of both clouds: lo starts at +3.4e38, hi at -3.4e38 (as ordered ints)
    int* box = reinterpret_cast<int*>(c.scal + kBox);
    CK(cudaMemsetAsync(box, 0x7F, kSortDims * sizeof(int), c.st));
    CK(cudaMemsetAsync(box + kSortDims, 0x80, kSortDims * sizeof(int), c.st));
    dim3 gx(reduce_blocks(p->n, c.sms), sdims), gy(reduce_blocks(p->m, c.sms), sdims);
    bbox_kernel<<<gx, 256, 0, c.st>>>(p->x, p->n, p->d, box, box + kSortDims);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    bbox_kernel<<<gy, 256, 0, c.st>>>(p->y, p->m, p->d, box, box + kSortDims);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  const bool wide = c.use_tc && tc_wide(c.L.Dtc);
  double* sum_x = wide ? c.tc_sums : c.scal + kSumX;
  double* sum_y = wide ? c.tc_sums + c.L.Dtc : c.scal + kSumY;
  if (wide) CK(cudaMemsetAsync(c.tc_sums, 0, 2 * c.L.Dtc * sizeof(double), c.st));
  if (c.use_tc) {
    unsigned* mx = reinterpret_cast<unsigned*>(c.scal + kMaxAbs);
    dim3 gx(reduce_blocks(p->n, c.sms), p->d), gy(reduce_blocks(p->m, c.sms), p->d);
    coord_stats_kernel<<<gx, 256, 0, c.st>>>(p->x, p->n, p->d, sum_x, mx);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    coord_stats_kernel<<<gy, 256, 0, c.st>>>(p->y, p->m, p->d, sum_y, mx);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  check_coords_kernel<<<reduce_blocks(p->n * p->d, c.sms), 256, 0, c.st>>>(
      p->x, p->n * p->d, flags_ptr(c.scal), reinterpret_cast<unsigned long long*>(c.scal + kHashX));
  CK(cudaGetLastError());
  g_launches.fetch_add(1, std::memory_order_relaxed);
  check_coords_kernel<<<reduce_blocks(p->m * p->d, c.sms), 256, 0, c.st>>>(
      p->y, p->m * p->d, flags_ptr(c.scal), reinterpret_cast<unsigned long long*>(c.scal + kHashY));
  CK(cudaGetLastError());
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (p->a) {
    reduce_weights_kernel<<<reduce_blocks(p->n, c.sms), 256, 0, c.st>>>(p->a, p->n, c.scal + kSumA,
                                                                       flags_ptr(c.scal));
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  if (p->b) {
    reduce_weights_kernel<<<reduce_blocks(p->m, c.sms), 256, 0, c.st>>>(p->b, p->m, c.scal + kSumB,
                                                                       flags_ptr(c.scal));
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  for (auto& pv : pots) {
    check_finite_kernel<<<reduce_blocks(pv.second, c.sms), 256, 0, c.st>>>(pv.first, pv.second,
                                                                          flags_ptr(c.scal));
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  double host[kBox + 3];  // through the bounding box (6 ints at kBox)
  unsigned long long memo[kSortMemoWords];
  std::vector<double> wide_sums(wide ? 2 * c.L.Dtc : 0);
  CK(cudaMemcpyAsync(host, c.scal, sizeof(host), cudaMemcpyDeviceToHost, c.st));
  CK(cudaMemcpyAsync(memo, c.scal + kSortMemo, sizeof(memo), cudaMemcpyDeviceToHost, c.st));
  if (wide)
    CK(cudaMemcpyAsync(wide_sums.data(), c.tc_sums, wide_sums.size() * sizeof(double),
                       cudaMemcpyDeviceToHost, c.st));
  CK(cudaStreamSynchronize(c.st));
  unsigned flags;
  memcpy(&flags, &host[kFlags], sizeof(unsigned));
  if (flags & 2u) return FS_ERR_NEGATIVE_WEIGHT;
  if (flags & (1u | 4u)) return FS_ERR_NONFINITE_INPUT;
  c.ma = p->a ? host[kSumA] : static_cast<double>(static_cast<float>(1.0 / p->n)) * p->n;
  c.mb = p->b ? host[kSumB] : static_cast<double>(static_cast<float>(1.0 / p->m)) * p->m;
  if (!(c.ma > 0.0) || !(c.mb > 0.0)) return FS_ERR_ZERO_MASS;
  if (std::fabs(c.ma - c.mb) > 1e-5 * std::max(c.ma, c.mb)) return FS_ERR_MASS_MISMATCH;

  if (c.L.sorted) {
    // Morton order on the first three coordinates over the common bounding box.
    int boxi[2 * kSortDims];
    memcpy(boxi, &host[kBox], sizeof(boxi));
    MortonFrame F{};
    F.dims = sdims;
    F.bits = sdims == 3 ? 10 : (sdims == 2 ? 16 : 30);
    for (int k = 0; k < sdims; ++k) {
      const float lo = ord_float(boxi[k]), hi = ord_float(boxi[kSortDims + k]);
      c.ctr[k] = 0.5f * (lo + hi);
      F.lo[k] = lo;
      F.scale[k] = hi > lo ? static_cast<float>(((1u << F.bits) - 1u) / (static_cast<double>(hi) - lo))
                           : 0.0f;
    }
    // The sort depends only on the coordinates (through them, on the frame). A workspace
    // keeps a record of its last sort: the shapes, both clouds' fingerprints, the frame and
    // where the permutations and codes lie; a call that matches it reuses them. (Any
    // permutation gives correct results; the order only decides how well screening works.)
    unsigned long long hx, hy;
    memcpy(&hx, &host[kHashX], sizeof(hx));
    memcpy(&hy, &host[kHashY], sizeof(hy));
    unsigned long long frame = static_cast<unsigned long long>(F.dims) | (static_cast<unsigned long long>(F.bits) << 8);
    for (int k = 0; k < 2 * kSortDims; ++k)
      frame = (frame * 0x100000001b3ull) ^ static_cast<unsigned>(boxi[k]);
    const SortMemo want{{kSortMagic, static_cast<unsigned long long>(p->n),
                         static_cast<unsigned long long>(p->m), static_cast<unsigned long long>(p->d),
                         hx, hy, c.L.off_perm_x, c.L.off_perm_y, c.L.off_code_x, c.L.off_code_y,
                         static_cast<unsigned long long>(c.L.sort_n), frame}};
    if (memcmp(want.v, memo, sizeof(memo)) != 0) {
      sort_cloud(p->x, p->n, p->d, F, c.sortkeys, c.L.sort_n, c.perm_x, c.code_x, c.st);
      sort_cloud(p->y, p->m, p->d, F, c.sortkeys, c.L.sort_n, c.perm_y, c.code_y, c.st);
      sort_memo_kernel<<<1, 32, 0, c.st>>>(
          reinterpret_cast<unsigned long long*>(c.scal + kSortMemo), want);
      CK(cudaGetLastError());
      g_launches.fetch_add(1, std::memory_order_relaxed);
    }
  } else {
    // this layout may overwrite where a sorted layout keeps its permutations
    CK(cudaMemsetAsync(c.scal + kSortMemo, 0, sizeof(unsigned long long), c.st));
  }
  const float wu_x = static_cast<float>(1.0 / p->n), wu_y = static_cast<float>(1.0 / p->m);
  FS_DISPATCH_D(c.L.D, launch_pack_d, p->x, p->n, p->d, p->a, wu_x, c.perm_x, c.kx, c.lwx, c.L.px,
                c.st);
  FS_DISPATCH_D(c.L.D, launch_pack_d, p->y, p->m, p->d, p->b, wu_y, c.perm_y, c.ky, c.lwy, c.L.py,
                c.st);
  if (c.L.sorted) {
    FS_DISPATCH_D(c.L.D, launch_tile_box_d, c.kx, p->n, c.L.px / kPairPad, c.box_x, c.gsum_x, c.st);
    FS_DISPATCH_D(c.L.D, launch_tile_box_d, c.ky, p->m, c.L.py / kPairPad, c.box_y, c.gsum_y, c.st);
  }
  if (c.use_tc) {
    // Centre on the common mean (the cost is translation invariant) and scale by a power of
    // two that puts the largest centred coordinate near 2^14, well inside fp16 range.
    TcCenter ctr{};
    double cmax = 0.0;
    if (wide) c.tc_ctr_host.assign(c.L.Dtc, 0.0);
    for (int k = 0; k < p->d; ++k) {
      const double sx = wide ? wide_sums[k] : host[kSumX + k];
      const double sy = wide ? wide_sums[c.L.Dtc + k] : host[kSumY + k];
      const double ck = (sx + sy) / static_cast<double>(p->n + p->m);
      if (wide)
        c.tc_ctr_host[k] = ck;
      else
        ctr.c[k] = ck;
      cmax = std::max(cmax, std::fabs(ck));
    }
    unsigned bits;
    memcpy(&bits, &host[kMaxAbs], sizeof(unsigned));
    float fmaxabs;
    memcpy(&fmaxabs, &bits, sizeof(float));
    const double bound = static_cast<double>(fmaxabs) + cmax;
    const double scale = bound > 0.0 ? std::exp2(std::floor(std::log2(16384.0 / bound))) : 1.0;
    c.c2 = static_cast<float>(2.0 * c.kappa / (scale * scale));
    c.tc_ctr = ctr;
    c.tc_scale = static_cast<float>(scale);
    c.tc_rkey = std::sqrt(static_cast<double>(p->d)) * bound;
    const float sc = static_cast<float>(scale);
    if (wide) {
      CK(cudaMemcpyAsync(c.tc_ctr_dev, c.tc_ctr_host.data(), c.L.Dtc * sizeof(double),
                         cudaMemcpyHostToDevice, c.st));
      const int kc = c.L.Dtc / kTcChunk;
      build_wide_image_kernel<<<static_cast<unsigned>(ceil_div(c.L.tx, 256)), 256, 0, c.st>>>(
          p->x, p->n, p->d, kc, c.tc_ctr_dev, sc, c.img_x, c.nrm_x, c.L.tx);
      CK(cudaGetLastError());
      build_wide_image_kernel<<<static_cast<unsigned>(ceil_div(c.L.ty, 256)), 256, 0, c.st>>>(
          p->y, p->m, p->d, kc, c.tc_ctr_dev, sc, c.img_y, c.nrm_y, c.L.ty);
      CK(cudaGetLastError());
      g_launches.fetch_add(2, std::memory_order_relaxed);
    } else switch (c.L.Dtc) {
      case 32:
        launch_image<32>(p->x, p->n, p->d, ctr, sc, c.img_x, c.nrm_x, c.L.tx, c.st);
        launch_image<32>(p->y, p->m, p->d, ctr, sc, c.img_y, c.nrm_y, c.L.ty, c.st);
        break;
      case 48:
        launch_image<48>(p->x, p->n, p->d, ctr, sc, c.img_x, c.nrm_x, c.L.tx, c.st);
        launch_image<48>(p->y, p->m, p->d, ctr, sc, c.img_y, c.nrm_y, c.L.ty, c.st);
        break;
      default:
        launch_image<64>(p->x, p->n, p->d, ctr, sc, c.img_x, c.nrm_x, c.L.tx, c.st);
        launch_image<64>(p->y, p->m, p->d, ctr, sc, c.img_y, c.nrm_y, c.L.ty, c.st);
        break;
    }
  }
  return FS_OK;
}

// Sets the key bias of one cloud from a potential (NULL = zero potential), in the form the
// next pass reads: the packed-key slot (FMA path) or the hy array (tensor-core path).
void set_bias(Ctx& c, bool cloud_x, const float* pot);

// prepare() followed by a zero-potential bias on both clouds in the tensor-core layout, so
// the padding columns of both hy arrays hold log2(0) before any pass reads them.
fs_status prepare_all(Ctx& c, const std::vector<std::pair<const float*, int64_t>>& pots,
                      bool need_tc) {
  const fs_status r = prepare(c, pots, need_tc);
  if (r != FS_OK || !c.use_tc) return r;
  set_bias(c, true, nullptr);
  set_bias(c, false, nullptr);
  return FS_OK;
}

void set_bias(Ctx& c, bool cloud_x, const float* pot) {
  if (c.use_tc) {
    const int64_t count = cloud_x ? c.p->n : c.p->m, pad = cloud_x ? c.L.tx : c.L.ty;
    tc_key_bias_kernel<<<static_cast<unsigned>(ceil_div(pad, 256)), 256, 0, c.st>>>(
        cloud_x ? c.hy_x : c.hy_y, count, pad, pot, cloud_x ? c.lwx : c.lwy,
        cloud_x ? c.nrm_x : c.nrm_y, c.kappa);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return;
  }
  if (cloud_x)
    FS_DISPATCH_D(c.L.D, launch_bias_d, c.kx, c.p->n, pot, c.perm_x, c.lwx, c.kappa, c.st)
  else
    FS_DISPATCH_D(c.L.D, launch_bias_d, c.ky, c.p->m, pot, c.perm_y, c.lwy, c.kappa, c.st)
  if (c.L.sorted) {
    // largest bias per tile, for the screening of the passes that take this cloud as keys
    FS_DISPATCH_D(c.L.D, launch_tile_hmax_d, cloud_x ? c.kx : c.ky, cloud_x ? c.p->n : c.p->m,
                  (cloud_x ? c.L.px : c.L.py) / kPairPad, cloud_x ? c.hmax_x : c.hmax_y,
                  cloud_x ? c.gsum_x : c.gsum_y, c.st);
  }
}

// One streaming pass with rows from cloud x (rows_x) or y, keys from the other cloud.
void run_pass_tc(Ctx& c, bool rows_x, int kind, const float* pot_in, float* pot_out,
                 float* marg_out, double* acc, float* lse_out = nullptr, int timed_kind = -1) {
  const fs_problem* p = c.p;
  const int64_t n_rows = rows_x ? p->n : p->m, n_keys = rows_x ? p->m : p->n;
  const TcPlan pl = make_tc_plan(n_rows, n_keys, c.L.Dtc, c.sms);
  PassParams P{};
  P.n_rows = n_rows;
  P.n_splits = pl.n_splits;
  P.rows_pad = pl.rows_pad;
  P.kind = kind;
  P.d_real = p->d;
  P.kappa = c.kappa;
  P.kappa_f = static_cast<float>(c.kappa);
  P.inv_kappa_f = static_cast<float>(1.0 / c.kappa);
  P.eps_ln2 = 1.0 / c.kappa;
  P.lw = rows_x ? c.lwx : c.lwy;
  P.w = rows_x ? p->a : p->b;
  P.w_uniform = static_cast<float>(1.0 / n_rows);
  P.pot_in = pot_in;
  P.pot_out = pot_out;
  P.marg_out = marg_out;
  P.acc = acc;
  P.part_m = c.part;
  P.part_l = c.part + static_cast<int64_t>(pl.n_splits) * pl.rows_pad;
  P.err = err_ptr(c.scal);
  P.hy_out = rows_x ? c.hy_x : c.hy_y;
  P.nrm = rows_x ? c.nrm_x : c.nrm_y;
  P.lse_out = lse_out;
  if (kind == kPot) {
    P.alpha = c.alpha;
    if (rows_x && c.defer_x) P.defer_h = c.defer;  // installed after the other pass
  }
  TcParams T{};
  T.row_img = rows_x ? c.img_x : c.img_y;
  T.key_img = rows_x ? c.img_y : c.img_x;
  T.key_hy = rows_x ? c.hy_y : c.hy_x;
  T.row_nrm = rows_x ? c.nrm_x : c.nrm_y;
  T.key_tiles = pl.key_tiles;
  T.tiles_per_split = pl.tiles_per_split;
  T.c2 = c.c2;
  T.kc = c.L.Dtc / kTcChunk;
  const double pairs = static_cast<double>(n_rows) * static_cast<double>(n_keys);
  int ti = c.timer->begin();
  launch_tc(c.L.Dtc, P, T, pl, c.st);
  c.timer->end(ti, timed_kind >= 0 ? timed_kind : (kind == kMarg ? kTMarg : kTLse), pairs);
  if (pl.n_splits > 1) {
    ti = c.timer->begin();
    FS_DISPATCH_D(c.L.D, launch_combine_d, P, false, c.st);
    c.timer->end(ti, kTCombine, 0.0);
  }
}

// An apply pass on the tensor cores (d > 16), rows from cloud x (rows_x) or y:
//   mode kApplyGrad: out = grad (n_rows x d) at the plan of (F(g), g), g carried by the keys;
//   mode kApplyPay:  out (n_rows x k, row stride out_stride) = P pay, pay (n_keys x k, row
//     stride pay_stride), P the plan of (pot_in, key potentials), or of (F(g), g) when pot_in
//     is NULL; channels go kPayChannels at a time;
//   mode kApplyDiff: out (n_rows x d) = sum_j P_ij (pay_j + (y_j - x_i).row_v_i)(y_j - x_i),
//     pay one value per key (dg), row_v (n_rows x d) one vector per row.
// First a potential-type pass writes every row's LSE2 (and, with pot_in, its plan mass),
// then the apply pass streams the keys again at those fixed offsets. With c.tc_reuse the
// first pre-pass of each direction serves every later apply pass of the call.
void run_apply_tc(Ctx& c, bool rows_x, int mode, const float* pot_in, const float* pay, int k,
                  int pay_stride, float* out, int out_stride, const float* row_v = nullptr) {
  const fs_problem* p = c.p;
  if (mode == kApplyGrad && tc_wide(c.L.Dtc)) {
    // Wide points: P y as a transport product at the plan of (F(g), g) (row masses w), in
    // the gradient's buffer, then grad = 2 (w x - P y) in place.
    const int64_t n_rows = rows_x ? p->n : p->m;
    run_apply_tc(c, rows_x, kApplyPay, nullptr, rows_x ? p->y : p->x, p->d, p->d, out, out_stride);
    grad_from_py_kernel<<<static_cast<unsigned>(ceil_div(n_rows * p->d, 256)), 256, 0, c.st>>>(
        rows_x ? p->x : p->y, rows_x ? p->a : p->b, static_cast<float>(1.0 / n_rows), out, n_rows,
        p->d, out);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return;
  }
  const int64_t n_rows = rows_x ? p->n : p->m, n_keys = rows_x ? p->m : p->n;
  const int tk = mode == kApplyGrad ? kTGrad : kTMarg;
  const int64_t half = std::max(c.L.tx, c.L.ty);
  float* lse = c.tc_lse + (rows_x ? 0 : half);
  float* mass = c.tc_mass + (rows_x ? 0 : half);
  const int dir = rows_x ? 0 : 1;
  if (!(c.tc_reuse && c.tc_valid[dir])) {
    if (pot_in)
      run_pass_tc(c, rows_x, kMarg, pot_in, nullptr, mass, nullptr, lse, tk);
    else
      run_pass_tc(c, rows_x, kLse, nullptr, nullptr, nullptr, nullptr, lse, tk);
    c.tc_valid[dir] = true;
  }
  const TcPlan pl = make_tc_plan(n_rows, n_keys, c.L.Dtc, c.sms);
  PassParams P{};
  P.n_rows = n_rows;
  P.n_splits = pl.n_splits;
  P.rows_pad = pl.rows_pad;
  P.kind = kGrad;
  P.d_real = p->d;
  P.kappa = c.kappa;
  P.kappa_f = static_cast<float>(c.kappa);
  P.inv_kappa_f = static_cast<float>(1.0 / c.kappa);
  P.eps_ln2 = 1.0 / c.kappa;
  P.w = rows_x ? p->a : p->b;
  P.w_uniform = static_cast<float>(1.0 / n_rows);
  P.part_l = c.part;
  P.part_a = c.part + static_cast<int64_t>(pl.n_splits) * pl.rows_pad;
  P.err = err_ptr(c.scal);
  TcParams T{};
  T.row_img = rows_x ? c.img_x : c.img_y;
  T.key_img = rows_x ? c.img_y : c.img_x;
  T.key_hy = rows_x ? c.hy_y : c.hy_x;
  T.row_nrm = rows_x ? c.nrm_x : c.nrm_y;
  T.key_tiles = pl.key_tiles;
  T.tiles_per_split = pl.tiles_per_split;
  T.c2 = c.c2;
  T.kc = c.L.Dtc / kTcChunk;
  TcApply A{};
  A.row_lse = lse;
  A.row_mass = pot_in ? mass : nullptr;
  A.x = rows_x ? p->x : p->y;
  A.inv_key_scale = 1.0f / c.tc_scale;
  memcpy(A.ctr, c.tc_ctr.c, sizeof(A.ctr));
  const double pairs = static_cast<double>(n_rows) * static_cast<double>(n_keys);
  if (mode == kApplyDiff) {
    const int64_t rpad = rows_x ? c.L.tx : c.L.ty, kpad = rows_x ? c.L.ty : c.L.tx;
    unsigned* vmax = reinterpret_cast<unsigned*>(c.scal + kVMax);
    unsigned* dgmax = reinterpret_cast<unsigned*>(c.scal + kDgMax);
    float* vinv = reinterpret_cast<float*>(c.scal + kVInv);
    CK(cudaMemsetAsync(vmax, 0, sizeof(unsigned), c.st));
    CK(cudaMemsetAsync(dgmax, 0, sizeof(unsigned), c.st));
    dg_prep_kernel<<<reduce_blocks(kpad, c.sms), 256, 0, c.st>>>(pay, n_keys, kpad, c.tc_dg, dgmax);
    CK(cudaGetLastError());
    pay_maxabs_kernel<<<reduce_blocks(n_rows * p->d, c.sms), 256, 0, c.st>>>(row_v, n_rows, p->d,
                                                                            p->d, vmax);
    CK(cudaGetLastError());
    const unsigned vb = static_cast<unsigned>(ceil_div(rpad, 256));
    const float rk = static_cast<float>(c.tc_rkey);
    const float* xr = rows_x ? p->x : p->y;
    switch (c.L.Dtc) {
      case 32:
        build_vrow_image_kernel<32><<<vb, 256, 0, c.st>>>(row_v, xr, n_rows, rpad, p->d, c.tc_ctr,
                                                          vmax, dgmax, rk, c.tc_vimg, c.tc_vrow, vinv);
        break;
      case 48:
        build_vrow_image_kernel<48><<<vb, 256, 0, c.st>>>(row_v, xr, n_rows, rpad, p->d, c.tc_ctr,
                                                          vmax, dgmax, rk, c.tc_vimg, c.tc_vrow, vinv);
        break;
      default:
        build_vrow_image_kernel<64><<<vb, 256, 0, c.st>>>(row_v, xr, n_rows, rpad, p->d, c.tc_ctr,
                                                          vmax, dgmax, rk, c.tc_vimg, c.tc_vrow, vinv);
        break;
    }
    CK(cudaGetLastError());
    g_launches.fetch_add(3, std::memory_order_relaxed);
    A.v_img = c.tc_vimg;
    A.v_row = c.tc_vrow;
    A.key_dg = c.tc_dg;
    A.v_inv_scale = vinv;
  }
  if (mode != kApplyPay) {
    A.out = out;
    A.out_stride = out_stride;
    int ti = c.timer->begin();
    launch_apply_tc(c.L.Dtc, mode, P, T, A, pl, c.st);
    c.timer->end(ti, tk, pairs);
    return;
  }
  unsigned* mx = reinterpret_cast<unsigned*>(c.scal + kPayMax);
  float* inv = reinterpret_cast<float*>(c.scal + kPayInv);
  const int64_t kpad = rows_x ? c.L.ty : c.L.tx;
  A.pay_img = c.tc_pay;
  A.pay_inv_scale = inv;
  for (int c0 = 0; c0 < k; c0 += kPayChannels) {
    const int kc = std::min(kPayChannels, k - c0);
    CK(cudaMemsetAsync(mx, 0, sizeof(unsigned), c.st));
    pay_maxabs_kernel<<<reduce_blocks(n_keys * kc, c.sms), 256, 0, c.st>>>(pay + c0, n_keys, kc,
                                                                          pay_stride, mx);
    CK(cudaGetLastError());
    build_pay_image_kernel<kPayChannels><<<static_cast<unsigned>(ceil_div(kpad, 256)), 256, 0,
                                           c.st>>>(pay + c0, n_keys, kpad, kc, pay_stride, mx,
                                                   c.tc_pay, inv);
    CK(cudaGetLastError());
    g_launches.fetch_add(2, std::memory_order_relaxed);
    A.out = out + c0;
    A.out_k = kc;
    A.out_stride = out_stride;
    int ti = c.timer->begin();
    launch_apply_tc(c.L.Dtc, mode, P, T, A, pl, c.st);
    c.timer->end(ti, tk, pairs);
  }
}

// A transport or Hessian-vector pass: what it accumulates, the streamed keys with their
// payload, the row vectors (kModeDiff) and where the results go.
struct PassExtra {
  int sel;
  const float* tile_keys;
  const float* row_v;
  float* out;
  int k, stride;
};

// Sorted FMA passes screen key tiles (see the kernel); `history` adds the bound from the
// rows' previous LSE2 and the keys' bias change, which exists from a solve's second iteration.
void run_pass(Ctx& c, bool rows_x, int kind, const float* pot_in, float* pot_out, float* marg_out,
              float* grad_out, double* acc, bool history = false, const PassExtra* ex = nullptr) {
  if (c.use_tc && kind != kGrad) {
    run_pass_tc(c, rows_x, kind, pot_in, pot_out, marg_out, acc);
    return;
  }
  if (c.use_tc && kind == kGrad && !ex) {
    run_apply_tc(c, rows_x, kApplyGrad, nullptr, nullptr, 0, 0, grad_out, c.p->d);
    return;
  }
  const fs_problem* p = c.p;
  // transport passes are planned (and their partials sized) like the gradient pass
  const bool grad = kind == kGrad || ex != nullptr;
  const int sel = ex ? ex->sel : (kind == kGrad ? kSelGrad : kSelLse);
  const int64_t n_rows = rows_x ? p->n : p->m;
  const int64_t key_pairs = rows_x ? c.L.py : c.L.px;
  const Plan pl = make_plan(n_rows, key_pairs, c.L.D, grad, c.sms);
  PassParams P{};
  if (ex) {
    P.tile_keys = ex->tile_keys;
    P.row_v = ex->row_v;
    P.acc_out = ex->out;
    P.acc_k = ex->k;
    P.acc_stride = ex->stride;
  }
  P.keys = rows_x ? c.ky : c.kx;
  P.qkeys = rows_x ? c.kx : c.ky;
  P.n_rows = n_rows;
  P.key_pairs = key_pairs;
  P.pairs_per_split = pl.pairs_per_split;
  P.tile_pairs = pl.tile_pairs;
  P.n_splits = pl.n_splits;
  P.rows_pad = pl.rows_pad;
  P.kind = kind;
  P.d_real = p->d;
  P.kappa = c.kappa;
  P.kappa_f = static_cast<float>(c.kappa);
  P.inv_kappa_f = static_cast<float>(1.0 / c.kappa);
  P.eps_ln2 = 1.0 / c.kappa;
  P.lw = rows_x ? c.lwx : c.lwy;
  P.w = rows_x ? p->a : p->b;
  P.w_uniform = static_cast<float>(1.0 / n_rows);
  P.pot_in = pot_in;
  P.pot_out = pot_out;
  P.marg_out = marg_out;
  P.grad_out = grad_out;
  P.acc = acc;
  P.part_m = c.part;
  P.part_l = c.part + static_cast<int64_t>(pl.n_splits) * pl.rows_pad;
  P.part_a = c.part + 2 * static_cast<int64_t>(pl.n_splits) * pl.rows_pad;
  P.err = err_ptr(c.scal);
  int* dmin_slots = reinterpret_cast<int*>(c.scal + kDmin);
  const int tk = grad ? kTGrad : (kind == kMarg ? kTMarg : kTLse);
  const QPlan q = make_qplan(pl, key_pairs, c.L.D, grad, c.sms, screening_live(c));
  if (c.L.sorted) {
    P.perm = rows_x ? c.perm_x : c.perm_y;
    P.evaluated = reinterpret_cast<unsigned long long*>(c.scal + kEval + tk);
    if (kind == kPot) {
      // this pass writes the query cloud's biases: record their change and its LSE2
      P.lse_out = rows_x ? c.lse_x : c.lse_y;
      P.alpha = c.alpha;
      if (rows_x && c.defer_x) {
        // installed, and its change recorded, after the other pass of the iteration: the
        // change recorded for x so far must survive until that pass has screened with it
        P.defer_h = c.defer;
      } else {
        P.dmin_out = dmin_slots + (rows_x ? 0 : 1);
        CK(cudaMemsetAsync(P.dmin_out, 0x7F, sizeof(int), c.st));
      }
    }
  }
  const double pairs = static_cast<double>(n_rows) * static_cast<double>(rows_x ? p->m : p->n);
  if (q.on) {
    const int64_t n_keys = rows_x ? p->m : p->n;
    const int64_t T = key_pairs / kPairPad, S = ceil_div(T, kSuper);
    P.key_tiles = static_cast<int32_t>(T);
    P.key_supers = static_cast<int32_t>(S);
    P.key_box = rows_x ? c.box_y : c.box_x;
    P.key_hmax = rows_x ? c.hmax_y : c.hmax_x;
    P.key_sbox = P.key_box + 2 * c.L.D * T;
    P.key_shmax = P.key_hmax + T;
    P.log2_keys = static_cast<float>(std::log2(static_cast<double>(n_keys)));
    P.skip_margin = kSkipBits + P.log2_keys;
    if (history && kind == kPot) {
      P.key_dmin = dmin_slots + (rows_x ? 1 : 0);
      P.lse_prev = rows_x ? c.lse_x : c.lse_y;
    }
    P.part_l = c.part + q.units_max * q.RB;
    P.part_a = c.part + 2 * q.units_max * q.RB;
    P.mask_words = q.mask_words;
    P.rb_rows = q.RB;
    P.kcount = c.kcount;
    P.unit_start = c.ustart;
    P.unit_rb = c.unit_rb;
    P.unit_j = c.unit_j;
    P.qscal = reinterpret_cast<const int*>(c.scal + kQueue);
    P.key_codes = rows_x ? c.code_y : c.code_x;
    P.row_codes = rows_x ? c.code_x : c.code_y;
    P.key_count = n_keys;
    // The first kAnchorRecords screens of each direction in a call evaluate the anchor tiles
    // and record each row's best key; later ones evaluate only that key.
    const int dir = rows_x ? 0 : 1;
    P.anchor_key = rows_x ? c.akey_x : c.akey_y;
    // the screen leaves each row's threshold; the pass then skips the 16-point groups of
    // kept tiles that no row of its block needs
    P.row_thr = c.rowthr;
    P.gsum = rows_x ? c.gsum_y : c.gsum_x;
    P.anchor_mode = c.anchor_records[dir] >= kAnchorRecords ? 2 : 1;
    if (P.anchor_mode == 1) ++c.anchor_records[dir];
    int ti = c.timer->begin();
    FS_DISPATCH_D(c.L.D, launch_screen_d, P, q.rb, c.kmask, c.kcount, c.st);
    plan_units_kernel<<<1, 1024, 0, c.st>>>(c.kcount, static_cast<int>(q.rb), q.budget, q.RB,
                                            c.ustart, c.unit_rb, c.unit_j,
                                            reinterpret_cast<int*>(c.scal + kQueue),
                                            reinterpret_cast<long long*>(c.scal + kKept),
                                            nullptr);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    c.timer->end(ti, kTScreen, 0.0);
    P.kmask = c.kmask;  // the pass counts the tiles each warp evaluates
    ti = c.timer->begin();
    FS_DISPATCH_D(c.L.D, launch_queue_d, P, q.units_max, sel, c.st);
    c.timer->end(ti, tk, pairs);
    ti = c.timer->begin();
    FS_DISPATCH_D(c.L.D, launch_combine_d, P, sel, c.st);
    c.timer->end(ti, kTCombine, 0.0);
  } else {
    int ti = c.timer->begin();
    FS_DISPATCH_D(c.L.D, launch_pass_d, P, pl, sel, c.st);
    c.timer->end(ti, tk, pairs);
    if (pl.n_splits > 1) {
      ti = c.timer->begin();
      FS_DISPATCH_D(c.L.D, launch_combine_d, P, sel, c.st);
      c.timer->end(ti, kTCombine, 0.0);
    }
  }
  if (screening_live(c) && kind == kPot && !(rows_x && c.defer_x)) {
    // largest bias per tile of the cloud just updated: the next pass screens against it (no
    // later pass of this call screens once screening is off)
    FS_DISPATCH_D(c.L.D, launch_tile_hmax_d, rows_x ? c.kx : c.ky, n_rows,
                  (rows_x ? c.L.px : c.L.py) / kPairPad, rows_x ? c.hmax_x : c.hmax_y,
                  rows_x ? c.gsum_x : c.gsum_y, c.st);
  }
}

// After a solve's first iteration: if the last screened pass (rows from x when rows_x, else
// from y) kept more than half of all (row block, key tile) pairs, screening cannot pay for
// its planning and merging, and the remaining passes of the call run unscreened.
void screening_probe(Ctx& c, bool rows_x) {
  const int64_t n_rows = rows_x ? c.p->n : c.p->m;
  const int64_t key_pairs = rows_x ? c.L.py : c.L.px;
  const Plan pl = make_plan(n_rows, key_pairs, c.L.D, false, c.sms);
  const QPlan q = make_qplan(pl, key_pairs, c.L.D, false, c.sms, screening_live(c));
  if (!q.on) return;
  long long kept = 0;
  CK(cudaMemcpyAsync(&kept, c.scal + kKept, sizeof(kept), cudaMemcpyDeviceToHost, c.st));
  CK(cudaStreamSynchronize(c.st));
  const double all = static_cast<double>(q.rb) * static_cast<double>(key_pairs / (kScreenTile / 2));
  if (static_cast<double>(kept) > 0.5 * all) c.no_screen = true;
}

// Drains the stream and reads the kernels' error word (after ORing in an armed injection).
fs_status finish(Ctx& c) {
  const unsigned inject = g_inject.exchange(0u);
  if (inject) {
    or_error_word_kernel<<<1, 32, 0, c.st>>>(err_ptr(c.scal), inject);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  double tail[kEval + 3 - kErr];
  CK(cudaMemcpyAsync(tail, c.scal + kErr, sizeof(tail), cudaMemcpyDeviceToHost, c.st));
  CK(cudaStreamSynchronize(c.st));
  unsigned err;
  unsigned long long evaluated[3];
  memcpy(&err, &tail[0], sizeof(unsigned));
  memcpy(evaluated, &tail[kEval - kErr], sizeof(evaluated));
  c.timer->collect(evaluated);
  return err ? FS_ERR_TIMEOUT : FS_OK;
}

template <typename F>
fs_status guarded(cudaStream_t st, F&& body) {
  try {
    return body();
  } catch (const CudaFail&) {
    cudaStreamSynchronize(st);
    cudaGetLastError();
    return FS_ERR_CUDA;
  }
}

fs_status begin(Ctx& c, const fs_problem* p, void* ws, size_t ws_bytes, fs_stream_t stream,
                int acc_ch = 0) {
  c.sms = num_sms_current();
  c.screen_on = g_screening.load();
  size_t need = 0;
  const fs_status s = check_common(p, ws, ws_bytes, &need, c.sms, acc_ch);
  if (s != FS_OK) return s;
  c.p = p;
  c.st = reinterpret_cast<cudaStream_t>(stream);
  c.L = make_layout(p->n, p->m, p->d, c.sms, acc_ch, p->cost == FS_COST_COSINE);
  c.kappa = 1.4426950408889634 / static_cast<double>(p->eps);
  carve(c, ws);
  return FS_OK;
}

// Symmetric schedule: install x's deferred biases once the y pass of the iteration has
// read the previous ones.
void apply_deferred_x(Ctx& c) {
  const int64_t n = c.p->n;
  if (c.use_tc) {
    CK(cudaMemcpyAsync(c.hy_x, c.defer, static_cast<size_t>(n) * sizeof(float),
                       cudaMemcpyDeviceToDevice, c.st));
    return;
  }
  int* dmin = reinterpret_cast<int*>(c.scal + kDmin);  // slot 0: x
  CK(cudaMemsetAsync(dmin, 0x7F, sizeof(int), c.st));
  FS_DISPATCH_D(c.L.D, launch_apply_bias_d, c.kx, c.defer, n, dmin, c.st);
  if (screening_live(c))
    FS_DISPATCH_D(c.L.D, launch_tile_hmax_d, c.kx, n, c.L.px / kPairPad, c.hmax_x, c.gsum_x, c.st);
}

// max(|P1 - a|_inf, |P^T 1 - b|_inf) at (f, g): two marginal passes, one read-back.
double check_marginal(Ctx& c, const float* f, const float* g) {
  CK(cudaMemsetAsync(c.scal + kAccRow, 0, 6 * sizeof(double), c.st));
  run_pass(c, true, kMarg, f, nullptr, nullptr, nullptr, c.scal + kAccRow);
  run_pass(c, false, kMarg, g, nullptr, nullptr, nullptr, c.scal + kAccCol);
  double acc[6];
  CK(cudaMemcpyAsync(acc, c.scal + kAccRow, sizeof(acc), cudaMemcpyDeviceToHost, c.st));
  CK(cudaStreamSynchronize(c.st));
  return std::max(acc[1], acc[4]);
}

// max(|f - f_prev|_inf, |g - g_prev|_inf), then prev <- current; one read-back.
double check_potential(Ctx& c, const float* f, const float* g) {
  unsigned* mb = reinterpret_cast<unsigned*>(c.scal + kPotChange);
  CK(cudaMemsetAsync(mb, 0, sizeof(unsigned), c.st));
  pot_change_kernel<<<reduce_blocks(c.p->n, c.sms), 256, 0, c.st>>>(f, c.fprev, c.p->n, mb);
  CK(cudaGetLastError());
  pot_change_kernel<<<reduce_blocks(c.p->m, c.sms), 256, 0, c.st>>>(g, c.gprev, c.p->m, mb);
  CK(cudaGetLastError());
  g_launches.fetch_add(2, std::memory_order_relaxed);
  unsigned bits = 0;
  CK(cudaMemcpyAsync(&bits, mb, sizeof(bits), cudaMemcpyDeviceToHost, c.st));
  CK(cudaStreamSynchronize(c.st));
  float v;
  memcpy(&v, &bits, sizeof(v));
  return static_cast<double>(v);
}

// out(i, c) = sum_j P_ij pay(j, c) for the rows of one cloud (rows_x: rows x, keys y), c < k,
// P the plan of (pot_in, key potentials) when pot_in is given, else of (F(g), g) (each row's
// mass is then its weight). The keys must carry their biases. Channels go 16 at a time.
void transport_pass(Ctx& c, bool rows_x, const float* pot_in, const float* pay, int k, int stride,
                    float* out, int out_stride, const float* row_v = nullptr) {
  if (c.use_tc) {
    if (row_v)
      run_apply_tc(c, rows_x, kApplyDiff, pot_in, pay, 1, stride, out, out_stride, row_v);
    else
      run_apply_tc(c, rows_x, kApplyPay, pot_in, pay, k, stride, out, out_stride);
    return;
  }
  const int64_t n_keys = rows_x ? c.p->m : c.p->n;
  const int64_t pairs = rows_x ? c.L.py : c.L.px;
  for (int c0 = 0; c0 < k; c0 += kTransportChannels) {
    const int kc = std::min(kTransportChannels, k - c0);
    const int np = row_v ? 1 : (kc == 1 ? 1 : (kc <= 4 ? 4 : 16));
    const int sel = row_v ? kSelDiff : (np == 1 ? kSelPay1 : (np == 4 ? kSelPay4 : kSelPay16));
    FS_DISPATCH_D(c.L.D, launch_payload_keys_d, rows_x ? c.ky : c.kx, n_keys, pairs, pay + c0, kc,
                  stride, rows_x ? c.perm_y : c.perm_x, c.paykeys, np, c.st);
    PassExtra ex{sel, c.paykeys, row_v, out + c0, row_v ? c.p->d : kc, out_stride};
    run_pass(c, rows_x, kMarg, pot_in, nullptr, nullptr, nullptr, nullptr, false, &ex);
  }
}

fs_status check_options(const fs_solve_options& o) {
  if (o.variant != FS_VARIANT_ALTERNATING && o.variant != FS_VARIANT_SYMMETRIC) return FS_ERR_OPTION;
  if (o.variant == FS_VARIANT_SYMMETRIC && !(o.alpha > 0.0f && o.alpha <= 1.0f)) return FS_ERR_OPTION;
  if (o.stop_mode == FS_STOP_FIXED) return o.n_iters < 1 ? FS_ERR_ITERS : FS_OK;
  if (o.stop_mode != FS_STOP_MARGINAL && o.stop_mode != FS_STOP_POTENTIAL) return FS_ERR_OPTION;
  if (o.stop_max_iter < 1 || o.stop_check_every < 1 || !(o.stop_tol >= 0.0)) return FS_ERR_OPTION;
  return FS_OK;
}

}  // namespace

// A stream the library captures graphs on: the caller's stream may be the legacy default
// stream, which cannot be captured. One per device, created on first use.
cudaStream_t capture_stream() {
  static std::mutex mu;
  static cudaStream_t streams[64] = {};
  int dev = 0;
  CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!streams[dev]) CK(cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking));
  return streams[dev];
}

// ---- small problems: the whole fixed-count solve in one cluster launch ----------------------

template <int D>
struct SmallKernel {
  static constexpr auto fn = small_solve_kernel<D>;
  // Launches one cluster of 16 CTAs (a non-portable size) if the device co-schedules it,
  // else of 8, 4, 2 or 1; the size that worked is remembered.
  static bool launch(const SmallParams& S, cudaStream_t st) {
    static int best = 0;  // 0: not tried yet; -1: unavailable
    static bool attr = false;
    if (!attr) {
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess ||
          cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kSmallSmemBudget)) != cudaSuccess) {
        cudaGetLastError();
        best = -1;
      }
      attr = true;
    }
    if (best < 0) return false;
    const size_t smem = small_smem_bytes(S.n, S.m, D);
    for (int cs = best ? best : kSmallMaxCluster; cs >= 1; cs /= 2) {
      cudaLaunchConfig_t cfg{};
      cudaLaunchAttribute at[1];
      cfg.gridDim = dim3(cs);
      cfg.blockDim = dim3(kSmallThreads);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = st;
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = cs;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      if (cudaLaunchKernelEx(&cfg, fn, S) == cudaSuccess) {
        best = cs;
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return true;
      }
      cudaGetLastError();  // a cluster this device cannot co-schedule: try a smaller one
    }
    best = -1;
    return false;
  }
};

// Whether the fixed-count alternating solve of this problem runs in one cluster launch:
// points of at most 16 coordinates, at most kSmallMaxPairs pairs, and both clouds staged in
// shared memory.
bool small_solve_fits(const fs_problem* p) {
  if (p->d > 16 || p->n * p->m > kSmallMaxPairs) return false;
  return small_smem_bytes(p->n, p->m, padded_dim(p->d)) <= kSmallSmemBudget;
}

// Runs the solve in one cluster launch; false (nothing launched) when the device cannot
// co-schedule a cluster for it.
bool run_small_solve(Ctx& c, int32_t n_iters, const float* g_init, float* f, float* g) {
  const fs_problem* p = c.p;
  SmallParams S{};
  S.x = p->x;
  S.y = p->y;
  S.a = p->a;
  S.b = p->b;
  S.wa = static_cast<float>(1.0 / p->n);
  S.wb = static_cast<float>(1.0 / p->m);
  S.g_init = g_init;
  S.f = f;
  S.g = g;
  S.n = static_cast<int32_t>(p->n);  // n * m <= kSmallMaxPairs
  S.m = static_cast<int32_t>(p->m);
  S.d = p->d;
  S.n_iters = n_iters;
  S.kappa = c.kappa;
  S.inv_kappa = 1.0 / c.kappa;
  S.err = err_ptr(c.scal);
  const double pairs = 2.0 * static_cast<double>(p->n) * static_cast<double>(p->m) * n_iters;
  const int ti = c.timer->begin();
  bool ok = false;
  switch (padded_dim(p->d)) {
    case 1: ok = SmallKernel<1>::launch(S, c.st); break;
    case 2: ok = SmallKernel<2>::launch(S, c.st); break;
    case 3: ok = SmallKernel<3>::launch(S, c.st); break;
    case 4: ok = SmallKernel<4>::launch(S, c.st); break;
    case 8: ok = SmallKernel<8>::launch(S, c.st); break;
    default: ok = SmallKernel<16>::launch(S, c.st); break;
  }
  c.timer->end(ti, kTLse, ok ? pairs : 0.0);
  return ok;
}

// Runs body() `count` times on c.st as one CUDA graph: body's launches are captured once
// (on the capture stream, so nothing runs during the capture) and the graph is replayed on
// the caller's stream, one launch instead of ~15 per replay. body() must issue the same
// launches with the same arguments every time and read nothing back. Returns false, having
// run nothing, when the capture is unavailable or refused one of body's calls; the caller
// then issues the work itself.
template <typename Body>
bool replay_as_graph(Ctx& c, int32_t count, Body&& body) {
  cudaStream_t cap = capture_stream();
  if (!cap) return false;
  const cudaStream_t user = c.st;
  if (cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const int64_t l0 = g_launches.load();
  cudaGraph_t graph = nullptr;
  c.st = cap;
  bool ok = true;
  try {
    body();
  } catch (const CudaFail&) {
    ok = false;  // a call the capture refused: nothing ran, so the caller issues it all
  }
  c.st = user;
  const int64_t per = g_launches.load() - l0;  // counted while capturing, not yet run
  g_launches.fetch_sub(per);
  if (cudaStreamEndCapture(cap, &graph) != cudaSuccess || !ok) {
    if (graph) cudaGraphDestroy(graph);
    cudaGetLastError();
    return false;
  }
  cudaGraphExec_t exec = nullptr;
  cudaError_t e = cudaGraphInstantiate(&exec, graph, 0);
  for (int32_t k = 0; e == cudaSuccess && k < count; ++k) {
    e = cudaGraphLaunch(exec, user);
    if (e == cudaSuccess) g_launches.fetch_add(per);
  }
  if (exec) {
    const cudaError_t se = cudaStreamSynchronize(user);  // the launches are done with it
    if (e == cudaSuccess) e = se;
    cudaGraphExecDestroy(exec);
  }
  cudaGraphDestroy(graph);
  CK(e);
  return true;
}

fs_status solve_impl(const fs_problem* p, const fs_solve_options* opt, float* f, float* g,
                     fs_solve_report* report, void* ws, size_t ws_bytes, fs_stream_t stream,
                     bool graphs_allowed = true) {
  Ctx c{};
  fs_status s = begin(c, p, ws, ws_bytes, stream);
  if (s != FS_OK) return s;
  if (!opt || !f || !g) return FS_ERR_NULL;
  const fs_solve_options o = *opt;
  if (!aligned4(f) || !aligned4(g) || !aligned4(o.g_init)) return FS_ERR_ALIGNMENT;
  s = check_options(o);
  if (s != FS_OK) return s;
  Timer timer(c.st);
  c.timer = &timer;
  return guarded(c.st, [&]() -> fs_status {
    std::vector<std::pair<const float*, int64_t>> pots;
    if (o.g_init) pots.push_back({o.g_init, p->m});
    fs_status r = prepare_all(c, pots, true);
    if (r != FS_OK) return r;
    const bool sym = o.variant == FS_VARIANT_SYMMETRIC;
    const bool fixed = o.stop_mode == FS_STOP_FIXED;
    const size_t fb = static_cast<size_t>(p->n) * sizeof(float);
    const size_t gb = static_cast<size_t>(p->m) * sizeof(float);
    if (sym || o.stop_mode == FS_STOP_POTENTIAL) {
      // the blend and the first potential check read the starting point f = 0, g = g_init
      if (o.g_init && o.g_init != g)
        CK(cudaMemcpyAsync(g, o.g_init, gb, cudaMemcpyDeviceToDevice, c.st));
      else if (!o.g_init)
        CK(cudaMemsetAsync(g, 0, gb, c.st));
      CK(cudaMemsetAsync(f, 0, fb, c.st));
    }
    if (o.stop_mode == FS_STOP_POTENTIAL) {
      CK(cudaMemsetAsync(c.fprev, 0, fb, c.st));
      CK(cudaMemcpyAsync(c.gprev, g, gb, cudaMemcpyDeviceToDevice, c.st));
    }
    if (!sym && fixed && small_solve_fits(c.p) && run_small_solve(c, o.n_iters, o.g_init, f, g)) {
      r = finish(c);
      if (report) {
        report->iters_run = o.n_iters;
        report->converged = -1;
        report->final_viol = NAN;
      }
      return r;
    }
    if (sym) set_bias(c, true, nullptr);  // x carries f = 0
    set_bias(c, false, o.g_init);
    c.alpha = sym ? o.alpha : 0.0f;
    const int32_t total = fixed ? o.n_iters : o.stop_max_iter;
    int32_t iters = 0, conv = fixed ? -1 : 0;
    double viol = NAN;
    // From the second iteration on every row has a previous LSE2 and the keys a recorded
    // bias change, so the passes can screen key tiles by history as well.
    auto iteration = [&](int32_t it) {
      c.defer_x = sym;
      run_pass(c, true, kPot, nullptr, f, nullptr, nullptr, nullptr, it > 1);   // f <- F(g)
      c.defer_x = false;
      run_pass(c, false, kPot, nullptr, g, nullptr, nullptr, nullptr, it > 1);  // g <- G(f)
      if (sym) apply_deferred_x(c);
    };
    // A fixed count issues the same launches in every iteration from the third on (the
    // screening decision is taken after the first, the screens record their anchor keys in
    // the first two): those run as replays of one CUDA graph, unless per-kernel timing is on
    // (it records events around each launch).
    constexpr int32_t kGraphFrom = kAnchorRecords + 1;
    const bool graphs = graphs_allowed && fixed && total > kGraphFrom && !c.timer->on();
    for (int32_t it = 1; it <= total; ++it) {
      if (graphs && it == kGraphFrom &&
          replay_as_graph(c, total - kGraphFrom + 1, [&] { iteration(kGraphFrom); })) {
        iters = total;
        break;
      }
      iteration(it);
      iters = it;
      if (it == 1 && total > 2) screening_probe(c, false);
      if (fixed || (it % o.stop_check_every != 0 && it != total)) continue;
      viol = o.stop_mode == FS_STOP_MARGINAL ? check_marginal(c, f, g) : check_potential(c, f, g);
      if (o.stop_mode == FS_STOP_MARGINAL ? viol <= o.stop_tol : viol < o.stop_tol) {
        conv = 1;
        break;
      }
    }
    c.alpha = 0.0f;
    r = finish(c);
    if (report) {
      report->iters_run = iters;
      report->converged = conv;
      report->final_viol = viol;
    }
    return r;
  });
}

fs_status transport_impl(const fs_problem* p, const float* f, const float* g, int32_t transpose,
                         int32_t k, const float* u, float* out, void* ws, size_t ws_bytes,
                         fs_stream_t stream) {
  Ctx c{};
  fs_status s = begin(c, p, ws, ws_bytes, stream, kTransportChannels);
  if (s != FS_OK) return s;
  if (!f || !g || !u || !out) return FS_ERR_NULL;
  if (!aligned4(f) || !aligned4(g) || !aligned4(u) || !aligned4(out)) return FS_ERR_ALIGNMENT;
  if (k < 1 || (transpose != 0 && transpose != 1)) return FS_ERR_OPTION;
  Timer timer(c.st);
  c.timer = &timer;
  return guarded(c.st, [&]() -> fs_status {
    fs_status r = prepare_all(c, {{f, p->n}, {g, p->m}}, true);
    if (r != FS_OK) return r;
    if (!transpose) {
      set_bias(c, false, g);  // keys y carry g; rows x carry f
      transport_pass(c, true, f, u, k, k, out, k);
    } else {
      set_bias(c, true, f);  // keys x carry f; rows y carry g
      transport_pass(c, false, g, u, k, k, out, k);
    }
    return finish(c);
  });
}

fs_status hvp_impl(const fs_problem* p, const float* g, const float* v, float* out,
                   const fs_hvp_options* opt, fs_hvp_report* report, void* ws, size_t ws_bytes,
                   fs_stream_t stream) {
  Ctx c{};
  fs_status s = begin(c, p, ws, ws_bytes, stream, kTransportChannels);
  if (s != FS_OK) return s;
  if (p->d > 64) return FS_ERR_UNSUPPORTED_D;  // no wide form of the difference pass
  if (p->cost != FS_COST_SQEUCLIDEAN) return FS_ERR_OPTION;
  if (!g || !v || !out) return FS_ERR_NULL;
  if (!aligned4(g) || !aligned4(v) || !aligned4(out)) return FS_ERR_ALIGNMENT;
  const int32_t max_iter = opt ? opt->cg_max_iter : 200;
  const double tol = opt ? opt->cg_tol : 1e-6;
  if (max_iter < 1 || !(tol >= 0.0)) return FS_ERR_OPTION;
  Timer timer(c.st);
  c.timer = &timer;
  return guarded(c.st, [&]() -> fs_status {
    fs_status r = prepare_all(c, {{g, p->m}}, true);
    if (r != FS_OK) return r;
    const int64_t n = p->n, m = p->m, nm = n + m;
    const int32_t d = p->d;
    // vectors
    float* ft = c.hvp;
    float* rv = ft + n;
    float* zu = rv + n;               // (df, dg) = z
    float* res = zu + nm;
    float* dir = res + nm;
    float* ap = dir + nm;
    float* prod = ap + nm;            // P w (n) then P^T u (m)
    float* grad = prod + nm;
    float* diffsum = grad + n * d;
    float* v2 = diffsum + n * d;
    float* colpay = v2 + n * d;        // (n, d + 2)
    float* coldata = colpay + n * (d + 2);  // (m, d + 2)
    float* csum = coldata + m * (d + 2);      // (m)
    float* zbest = csum + m;                  // (n + m), ends at hvp_floats(n, m, d) - 64
    double* dots = c.scal + kCgDots;
    const unsigned blk = static_cast<unsigned>(ceil_div(nm, 256));
    const float a_uni = static_cast<float>(1.0 / n);
    auto launched = [](int k) { g_launches.fetch_add(k, std::memory_order_relaxed); };
    auto read = [&](double* h, int count) {
      CK(cudaMemcpyAsync(h, dots, count * sizeof(double), cudaMemcpyDeviceToHost, c.st));
      CK(cudaStreamSynchronize(c.st));
    };
    // 1. keys y carry g; ft = F(g) gives keys x their biases kappa ft + log2 a
    set_bias(c, false, g);
    run_pass(c, true, kPot, nullptr, ft, nullptr, nullptr, nullptr);
    // From here on every bias is fixed: the tensor-core apply passes compute each
    // direction's row offsets once.
    c.tc_reuse = true;
    // 2. the gradient at the plan of (ft, g), r and the column pass's payload
    run_pass(c, true, kGrad, nullptr, nullptr, nullptr, grad, nullptr);
    hvp_row_prep_kernel<<<static_cast<unsigned>(ceil_div(n, 256)), 256, 0, c.st>>>(
        p->x, v, grad, n, d, c.ctr[0], c.ctr[1], c.ctr[2], res, colpay);
    CK(cudaGetLastError());
    transport_pass(c, false, g, colpay, d + 2, d + 2, coldata, d + 2);  // column sums and data
    hvp_col_rhs_kernel<<<static_cast<unsigned>(ceil_div(m, 256)), 256, 0, c.st>>>(
        p->y, coldata, m, d, c.ctr[0], c.ctr[1], c.ctr[2], res + n, csum);
    CK(cudaGetLastError());
    launched(2);
    // 3. conjugate gradients on [diag(P1) P; P^T diag(P^T 1)] z = (r, s), from z = 0, with
    //    the gauge direction (1, -1) removed from the right-hand side
    CK(cudaMemsetAsync(dots, 0, 4 * sizeof(double), c.st));
    cg_split_sum_kernel<<<reduce_blocks(nm, c.sms), 256, 0, c.st>>>(res, n, m, dots);
    cg_project_kernel<<<blk, 256, 0, c.st>>>(res, n, m, dots);
    CK(cudaMemsetAsync(zu, 0, nm * sizeof(float), c.st));
    CK(cudaMemcpyAsync(dir, res, nm * sizeof(float), cudaMemcpyDeviceToDevice, c.st));
    cg_dot_kernel<<<reduce_blocks(nm, c.sms), 256, 0, c.st>>>(res, res, nm, dots + 2);
    CK(cudaGetLastError());
    launched(3);
    double h[4];
    read(h, 4);
    const double bb = h[2];
    double rr = bb;
    int32_t it = 0;
    // the iterate with the smallest residual so far (z = 0 to begin with)
    constexpr int32_t kCgPatience = 50;
    double best = bb;
    int32_t best_it = 0;
    CK(cudaMemsetAsync(zbest, 0, nm * sizeof(float), c.st));
    while (it < max_iter && rr > tol * tol * bb && rr > 0.0) {
      transport_pass(c, true, nullptr, dir + n, 1, 1, prod, 1);      // P w
      transport_pass(c, false, g, dir, 1, 1, prod + n, 1);           // P^T u
      cg_apply_kernel<<<blk, 256, 0, c.st>>>(dir, p->a, a_uni, csum, prod, prod + n, n, m, ap);
      CK(cudaMemsetAsync(dots, 0, 2 * sizeof(double), c.st));
      cg_dot_kernel<<<reduce_blocks(nm, c.sms), 256, 0, c.st>>>(dir, ap, nm, dots);
      CK(cudaGetLastError());
      launched(2);
      read(h, 1);
      if (!(h[0] > 0.0)) break;
      const double alpha = rr / h[0];
      cg_step_kernel<<<blk, 256, 0, c.st>>>(zu, res, dir, ap, nm, static_cast<float>(alpha));
      cg_dot_kernel<<<reduce_blocks(nm, c.sms), 256, 0, c.st>>>(res, res, nm, dots + 1);
      CK(cudaGetLastError());
      launched(2);
      read(h, 2);
      const double rr_new = h[1];
      cg_dir_kernel<<<blk, 256, 0, c.st>>>(dir, res, nm, static_cast<float>(rr_new / rr));
      CK(cudaGetLastError());
      launched(1);
      rr = rr_new;
      ++it;
      if (rr < best) {
        best = rr;
        best_it = it;
        CK(cudaMemcpyAsync(zbest, zu, nm * sizeof(float), cudaMemcpyDeviceToDevice, c.st));
      } else if (it - best_it >= kCgPatience) {
        break;
      }
    }
    // 4. the difference pass with payload dg and row vectors 2 v, then the combination
    scale_kernel<<<static_cast<unsigned>(ceil_div(n * d, 256)), 256, 0, c.st>>>(v, n * d, 2.0f, v2);
    CK(cudaGetLastError());
    launched(1);
    transport_pass(c, true, nullptr, zbest + n, 1, 1, diffsum, d, v2);
    hvp_final_kernel<<<static_cast<unsigned>(ceil_div(n * d, 256)), 256, 0, c.st>>>(
        v, p->a, a_uni, zbest, grad, diffsum, n, d, 2.0 / static_cast<double>(p->eps), out);
    CK(cudaGetLastError());
    launched(1);
    r = finish(c);
    if (report) {
      report->cg_iters = it;
      report->cg_rel_residual = bb > 0.0 ? std::sqrt(best / bb) : 0.0;
    }
    return r;
  });
}

// ---------------- entry points ----------------

fs_status potentials_impl(const fs_problem* p, int32_t n_iters, const float* g_init, float* f,
                          float* g, void* ws, size_t ws_bytes, fs_stream_t stream,
                          bool graphs_allowed = true) {
  fs_solve_options o{};
  o.n_iters = n_iters;
  o.variant = FS_VARIANT_ALTERNATING;
  o.stop_mode = FS_STOP_FIXED;
  o.g_init = g_init;
  return solve_impl(p, &o, f, g, nullptr, ws, ws_bytes, stream, graphs_allowed);
}

// Records a CUDA error of another translation unit of the library for fs_last_cuda_error.
void record_cuda_error(const char* what, cudaError_t e) {
  snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace fs

extern "C" {

const char* fs_status_string(fs_status s) {
  switch (s) {
    case FS_OK: return "FS_OK";
    case FS_ERR_NULL: return "FS_ERR_NULL: a required pointer is NULL";
    case FS_ERR_SHAPE: return "FS_ERR_SHAPE: n, m and d must be >= 1";
    case FS_ERR_EPS: return "FS_ERR_EPS: eps must be finite and > 0";
    case FS_ERR_ITERS: return "FS_ERR_ITERS: n_iters must be >= 1";
    case FS_ERR_NEGATIVE_WEIGHT: return "FS_ERR_NEGATIVE_WEIGHT: weights must be finite and >= 0";
    case FS_ERR_NONFINITE_INPUT: return "FS_ERR_NONFINITE_INPUT: a coordinate or potential is not finite";
    case FS_ERR_MASS_MISMATCH: return "FS_ERR_MASS_MISMATCH: sum(a) and sum(b) differ by more than 1e-5 relative";
    case FS_ERR_ZERO_MASS: return "FS_ERR_ZERO_MASS: the total mass is zero";
    case FS_ERR_UNSUPPORTED_D: return "FS_ERR_UNSUPPORTED_D: d exceeds FS_MAX_D";
    case FS_ERR_WORKSPACE: return "FS_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case FS_ERR_TIMEOUT: return "FS_ERR_TIMEOUT: a kernel's bounded wait expired";
    case FS_ERR_CUDA: return "FS_ERR_CUDA: a CUDA runtime call failed";
    case FS_ERR_OPTION: return "FS_ERR_OPTION: a solve option is out of range";
    case FS_ERR_ALIGNMENT: return "FS_ERR_ALIGNMENT: device pointers must be 4-byte aligned";
    case FS_ERR_DEVICE_MEMORY:
      return "FS_ERR_DEVICE_MEMORY: the device could not commit the library's static scratch array";
  }
  return "unknown fs_status";
}

const char* fs_last_cuda_error(void) { return fs::g_cuda_err; }

size_t fs_workspace_bytes(const fs_problem* p) {
  if (!fs::shape_ok(p) || p->d > FS_MAX_D) return 0;
  return fs::make_layout(p->n, p->m, p->d, fs::num_sms_current(), 0,
                         p->cost == FS_COST_COSINE).total;
}

fs_status fs_potentials(const fs_problem* p, int32_t n_iters, const float* g_init, float* f,
                        float* g, void* ws, size_t ws_bytes, fs_stream_t stream) {
  return fs::potentials_impl(p, n_iters, g_init, f, g, ws, ws_bytes, stream);
}

fs_status fs_solve(const fs_problem* p, const fs_solve_options* opt, float* f, float* g,
                   fs_solve_report* report, void* ws, size_t ws_bytes, fs_stream_t stream) {
  return fs::solve_impl(p, opt, f, g, report, ws, ws_bytes, stream);
}

namespace {
// The two self problems of the divergence: (x, x, a, a) and (y, y, b, b).
void self_problems(const fs_problem* p, fs_problem* pxx, fs_problem* pyy) {
  *pxx = *p;
  pxx->y = p->x;
  pxx->b = p->a;
  pxx->m = p->n;
  *pyy = *p;
  pyy->x = p->y;
  pyy->a = p->b;
  pyy->n = p->m;
}
// The problem with the clouds' roles swapped.
fs_problem transposed(const fs_problem* p) {
  fs_problem t = *p;
  t.x = p->y;
  t.y = p->x;
  t.a = p->b;
  t.b = p->a;
  t.n = p->m;
  t.m = p->n;
  return t;
}
// Inner workspace of the divergence (the largest of its three problems), then its vectors:
// six potentials, two gradient buffers, three costs.
size_t divergence_inner_bytes(const fs_problem* p) {
  fs_problem pxx, pyy;
  self_problems(p, &pxx, &pyy);
  return std::max({fs_workspace_bytes(p), fs_workspace_bytes(&pxx), fs_workspace_bytes(&pyy)});
}
size_t divergence_tail_bytes(const fs_problem* p) {
  const size_t n = static_cast<size_t>(p->n), m = static_cast<size_t>(p->m),
               d = static_cast<size_t>(p->d);
  return fs::align_up((3 * n + 3 * m) * sizeof(float)) + fs::align_up(2 * std::max(n, m) * d * 4) +
         fs::align_up(3 * sizeof(double));
}
}  // namespace

size_t fs_divergence_workspace_bytes(const fs_problem* p) {
  if (!fs::shape_ok(p) || p->d > FS_MAX_D) return 0;
  return divergence_inner_bytes(p) + divergence_tail_bytes(p);
}

fs_status fs_divergence(const fs_problem* p, const fs_solve_options* opt, double* value,
                        float* grad_x, float* grad_y, void* ws, size_t ws_bytes,
                        fs_stream_t stream) {
  using namespace fs;
  if (!p || !opt || !value) return FS_ERR_NULL;
  if (!shape_ok(p)) return FS_ERR_SHAPE;
  if (p->d > FS_MAX_D) return FS_ERR_UNSUPPORTED_D;
  if ((reinterpret_cast<uintptr_t>(value) & 7u) || !aligned4(grad_x) || !aligned4(grad_y))
    return FS_ERR_ALIGNMENT;
  const size_t inner = divergence_inner_bytes(p);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 ||
      ws_bytes < inner + divergence_tail_bytes(p))
    return FS_ERR_WORKSPACE;
  const int64_t n = p->n, m = p->m, d = p->d;
  unsigned char* tail = static_cast<unsigned char*>(ws) + inner;
  float* fxy = reinterpret_cast<float*>(tail);
  float* gxy = fxy + n;
  float* fxx = gxy + m;
  float* gxx = fxx + n;
  float* fyy = gxx + n;
  float* gyy = fyy + m;
  float* tmp1 = reinterpret_cast<float*>(tail + align_up((3 * n + 3 * m) * sizeof(float)));
  float* tmp2 = tmp1 + std::max(n, m) * d;
  double* costs = reinterpret_cast<double*>(
      tail + align_up((3 * n + 3 * m) * sizeof(float)) +
      align_up(2 * static_cast<size_t>(std::max(n, m) * d) * 4));
  fs_problem pxx, pyy;
  self_problems(p, &pxx, &pyy);
  const fs_problem pyx = transposed(p);
  fs_solve_options o = *opt;
  o.g_init = nullptr;  // the three problems start alike
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  fs_status s;
  if ((s = solve_impl(p, &o, fxy, gxy, nullptr, ws, inner, stream)) != FS_OK) return s;
  if ((s = solve_impl(&pxx, &o, fxx, gxx, nullptr, ws, inner, stream)) != FS_OK) return s;
  if ((s = solve_impl(&pyy, &o, fyy, gyy, nullptr, ws, inner, stream)) != FS_OK) return s;
  if ((s = fs_cost(p, fxy, gxy, costs, ws, inner, stream)) != FS_OK) return s;
  if ((s = fs_cost(&pxx, fxx, gxx, costs + 1, ws, inner, stream)) != FS_OK) return s;
  if ((s = fs_cost(&pyy, fyy, gyy, costs + 2, ws, inner, stream)) != FS_OK) return s;
  divergence_finish_kernel<<<1, 32, 0, st>>>(costs, value);
  if (cudaGetLastError() != cudaSuccess) return FS_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  // grad_x S = grad_x OT(x, y) - (the self problem's gradients from both sides) / 2
  if (grad_x) {
    if ((s = fs_grad_x(p, gxy, grad_x, ws, inner, stream)) != FS_OK) return s;
    if ((s = fs_grad_x(&pxx, gxx, tmp1, ws, inner, stream)) != FS_OK) return s;
    if ((s = fs_grad_x(&pxx, fxx, tmp2, ws, inner, stream)) != FS_OK) return s;
    sub_half_sum_kernel<<<static_cast<unsigned>(ceil_div(n * d, 256)), 256, 0, st>>>(grad_x, tmp1,
                                                                                     tmp2, n * d);
    if (cudaGetLastError() != cudaSuccess) return FS_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  if (grad_y) {
    if ((s = fs_grad_x(&pyx, fxy, grad_y, ws, inner, stream)) != FS_OK) return s;
    if ((s = fs_grad_x(&pyy, gyy, tmp1, ws, inner, stream)) != FS_OK) return s;
    if ((s = fs_grad_x(&pyy, fyy, tmp2, ws, inner, stream)) != FS_OK) return s;
    sub_half_sum_kernel<<<static_cast<unsigned>(ceil_div(m * d, 256)), 256, 0, st>>>(grad_y, tmp1,
                                                                                     tmp2, m * d);
    if (cudaGetLastError() != cudaSuccess) return FS_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  return FS_OK;
}

namespace {
// The coarse stage's problems: the cell clouds (cx, ca; cy, cb) and the lift problem, fine y
// against the x cells; cells per cloud, and the tail of the workspace after the largest
// inner workspace of the fine, cell and lift problems.
struct Multiscale {
  int64_t ncx, ncy;
  fs_problem cells, lift;
  size_t inner, tail;
  float *cx, *cy, *ca, *cb, *fc, *gc, *gl, *tmp;
};

Multiscale multiscale_layout(const fs_problem* p, int cell_points, unsigned char* ws) {
  Multiscale M{};
  M.ncx = fs::ceil_div(p->n, cell_points);
  M.ncy = fs::ceil_div(p->m, cell_points);
  const int64_t d = p->d;
  M.cells = *p;
  M.cells.n = M.ncx;
  M.cells.m = M.ncy;
  M.lift = *p;  // rows: the fine y; keys: the x cells
  M.lift.n = p->m;
  M.lift.m = M.ncx;
  M.inner = std::max({fs_workspace_bytes(p), fs_workspace_bytes(&M.cells), fs_workspace_bytes(&M.lift)});
  size_t o = M.inner;
  auto take = [&](int64_t floats) {
    float* ptr = ws ? reinterpret_cast<float*>(ws + o) : nullptr;
    o = fs::align_up(o + static_cast<size_t>(floats) * sizeof(float));
    return ptr;
  };
  M.cx = take(M.ncx * d);
  M.cy = take(M.ncy * d);
  M.ca = take(M.ncx);
  M.cb = take(M.ncy);
  M.fc = take(M.ncx);
  M.gc = take(M.ncy);
  M.gl = take(p->m);
  M.tmp = take(M.ncx);
  M.tail = o - M.inner;
  M.cells.x = M.cx;
  M.cells.y = M.cy;
  M.cells.a = M.ca;
  M.cells.b = M.cb;
  M.lift.x = p->y;
  M.lift.y = M.cx;
  M.lift.a = p->b;
  M.lift.b = M.ca;
  return M;
}
}  // namespace

size_t fs_multiscale_workspace_bytes(const fs_problem* p, int32_t cell_points) {
  if (!fs::shape_ok(p) || p->d > 16 || cell_points < 1 || cell_points > fs::kScreenTile) return 0;
  const Multiscale M = multiscale_layout(p, cell_points, nullptr);
  return M.inner + M.tail;
}

fs_status fs_solve_multiscale(const fs_problem* p, const fs_solve_options* opt,
                              const fs_multiscale_options* mo, float* f, float* g,
                              fs_multiscale_report* report, void* ws, size_t ws_bytes,
                              fs_stream_t stream) {
  using namespace fs;
  if (!p || !opt || !mo || !f || !g) return FS_ERR_NULL;
  if (!shape_ok(p)) return FS_ERR_SHAPE;
  if (p->d > 16) return FS_ERR_UNSUPPORTED_D;
  if (p->cost != FS_COST_SQEUCLIDEAN) return FS_ERR_OPTION;
  fs_status s = check_options(*opt);
  if (s != FS_OK) return s;
  if (mo->coarse_iters < 1 || mo->max_rounds < 1 || !(mo->lift_tol >= 0.0) ||
      !(mo->lift_shrink > 0.0 && mo->lift_shrink <= 1.0) || mo->cell_points < 1 ||
      mo->cell_points > kScreenTile)
    return FS_ERR_OPTION;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return FS_ERR_WORKSPACE;
  const Multiscale M = multiscale_layout(p, mo->cell_points, static_cast<unsigned char*>(ws));
  if (ws_bytes < M.inner + M.tail) return FS_ERR_WORKSPACE;
  // cells of both clouds, from their Morton-sorted packed copies
  {
    Ctx c{};
    s = begin(c, p, ws, M.inner, stream);
    if (s != FS_OK) return s;
    Timer timer(c.st);
    c.timer = &timer;
    s = guarded(c.st, [&]() -> fs_status {
      const fs_status r = prepare_all(c, {}, false);
      if (r != FS_OK) return r;
      FS_DISPATCH_D(c.L.D, launch_cells_d, c.kx, p->n, p->d, p->a,
                    static_cast<float>(1.0 / p->n), c.perm_x, mo->cell_points, M.cx, M.ca, M.ncx,
                    c.st);
      FS_DISPATCH_D(c.L.D, launch_cells_d, c.ky, p->m, p->d, p->b,
                    static_cast<float>(1.0 / p->m), c.perm_y, mo->cell_points, M.cy, M.cb, M.ncy,
                    c.st);
      return finish(c);
    });
    if (s != FS_OK) return s;
  }
  // rounds on the cells, each followed by a lift and its check
  fs_solve_options co{};
  co.n_iters = mo->coarse_iters;
  co.variant = FS_VARIANT_ALTERNATING;
  co.stop_mode = FS_STOP_FIXED;
  fs_solve_options chk{};
  chk.variant = FS_VARIANT_ALTERNATING;
  chk.stop_mode = FS_STOP_MARGINAL;
  chk.stop_max_iter = 1;
  chk.stop_check_every = 1;
  chk.stop_tol = 0.0;
  chk.g_init = M.gl;
  int32_t rounds = 0;
  double viol = NAN, prev = NAN;
  for (int32_t r = 1; r <= mo->max_rounds; ++r) {
    co.g_init = r == 1 ? nullptr : M.gc;  // continue from the last round
    if ((s = solve_impl(&M.cells, &co, M.fc, M.gc, nullptr, ws, M.inner, stream)) != FS_OK) return s;
    // lift: g_j = G(f_cells)(y_j), the f-update of the problem (y, x cells) from f_cells
    if ((s = potentials_impl(&M.lift, 1, M.fc, M.gl, M.tmp, ws, M.inner, stream)) != FS_OK)
      return s;
    fs_solve_report cr{};
    if ((s = solve_impl(p, &chk, f, g, &cr, ws, M.inner, stream)) != FS_OK) return s;
    rounds = r;
    viol = cr.final_viol;
    const bool shrank_little = r > 1 && !(viol < mo->lift_shrink * prev);
    if (viol <= mo->lift_tol || shrank_little) break;
    prev = viol;
  }
  // the fine stage from the accepted lift
  fs_solve_options fo = *opt;
  fo.g_init = M.gl;
  fs_solve_report fr{};
  if ((s = solve_impl(p, &fo, f, g, &fr, ws, M.inner, stream)) != FS_OK) return s;
  if (report) {
    report->rounds = rounds;
    report->coarse_iters = rounds * mo->coarse_iters;
    report->lift_viol = viol;
    report->fine = fr;
  }
  return FS_OK;
}

size_t fs_transport_workspace_bytes(const fs_problem* p) {
  if (!fs::shape_ok(p) || p->d > FS_MAX_D) return 0;
  return fs::make_layout(p->n, p->m, p->d, fs::num_sms_current(), fs::kTransportChannels,
                         p->cost == FS_COST_COSINE).total;
}

fs_status fs_transport_apply(const fs_problem* p, const float* f, const float* g,
                             int32_t transpose, int32_t k, const float* u, float* out, void* ws,
                             size_t ws_bytes, fs_stream_t stream) {
  return fs::transport_impl(p, f, g, transpose, k, u, out, ws, ws_bytes, stream);
}

fs_status fs_hvp(const fs_problem* p, const float* g, const float* v, float* out,
                 const fs_hvp_options* opt, fs_hvp_report* report, void* ws, size_t ws_bytes,
                 fs_stream_t stream) {
  return fs::hvp_impl(p, g, v, out, opt, report, ws, ws_bytes, stream);
}

fs_status fs_grad_x(const fs_problem* p, const float* g, float* grad_x, void* ws, size_t ws_bytes,
                    fs_stream_t stream) {
  using namespace fs;
  Ctx c{};
  fs_status s = begin(c, p, ws, ws_bytes, stream);
  if (s != FS_OK) return s;
  if (!g || !grad_x) return FS_ERR_NULL;
  if (!aligned4(g) || !aligned4(grad_x)) return FS_ERR_ALIGNMENT;
  Timer timer(c.st);
  c.timer = &timer;
  return guarded(c.st, [&]() -> fs_status {
    fs_status r = prepare_all(c, {{g, p->m}}, true);
    if (r != FS_OK) return r;
    set_bias(c, false, g);
    run_pass(c, true, kGrad, nullptr, nullptr, nullptr, grad_x, nullptr);
    if (p->cost == FS_COST_COSINE) {
      cosine_grad_kernel<<<static_cast<unsigned>(ceil_div(p->n, 256)), 256, 0, c.st>>>(
          p->x, p->n, p->d, grad_x);
      CK(cudaGetLastError());
      g_launches.fetch_add(1, std::memory_order_relaxed);
    }
    return finish(c);
  });
}

fs_status fs_marginal_residual(const fs_problem* p, const float* f, const float* g, double* out,
                               float* row_marg, float* col_marg, void* ws, size_t ws_bytes,
                               fs_stream_t stream) {
  using namespace fs;
  Ctx c{};
  fs_status s = begin(c, p, ws, ws_bytes, stream);
  if (s != FS_OK) return s;
  if (!f || !g || !out) return FS_ERR_NULL;
  if (!aligned4(f) || !aligned4(g) || !aligned4(row_marg) || !aligned4(col_marg) ||
      (reinterpret_cast<uintptr_t>(out) & 7u))
    return FS_ERR_ALIGNMENT;
  Timer timer(c.st);
  c.timer = &timer;
  return guarded(c.st, [&]() -> fs_status {
    fs_status r = prepare_all(c, {{f, p->n}, {g, p->m}}, true);
    if (r != FS_OK) return r;
    set_bias(c, false, g);  // keys y carry g: row pass gives F(g)
    set_bias(c, true, f);   // keys x carry f: column pass gives G(f)
    run_pass(c, true, kMarg, f, nullptr, row_marg, nullptr, c.scal + kAccRow);
    run_pass(c, false, kMarg, g, nullptr, col_marg, nullptr, c.scal + kAccCol);
    residual_finish_kernel<<<1, 32, 0, c.st>>>(c.scal + kAccRow, c.scal + kAccCol, out);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return finish(c);
  });
}

fs_status fs_cost(const fs_problem* p, const float* f, const float* g, double* out, void* ws,
                  size_t ws_bytes, fs_stream_t stream) {
  using namespace fs;
  Ctx c{};
  fs_status s = begin(c, p, ws, ws_bytes, stream);
  if (s != FS_OK) return s;
  if (!f || !g || !out) return FS_ERR_NULL;
  if (!aligned4(f) || !aligned4(g) || (reinterpret_cast<uintptr_t>(out) & 7u))
    return FS_ERR_ALIGNMENT;
  Timer timer(c.st);
  c.timer = &timer;
  return guarded(c.st, [&]() -> fs_status {
    fs_status r = prepare_all(c, {{f, p->n}, {g, p->m}}, true);
    if (r != FS_OK) return r;
    set_bias(c, true, f);  // keys x carry f: column pass gives c_j = sum_i P_ij
    run_pass(c, false, kMarg, g, nullptr, nullptr, nullptr, c.scal + kAccCol);
    dot_kernel<<<reduce_blocks(p->n, c.sms), 256, 0, c.st>>>(f, p->a, static_cast<float>(1.0 / p->n),
                                                            p->n, c.scal + kDotFA);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    dot_kernel<<<reduce_blocks(p->m, c.sms), 256, 0, c.st>>>(g, p->b, static_cast<float>(1.0 / p->m),
                                                            p->m, c.scal + kDotGB);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    cost_finish_kernel<<<1, 32, 0, c.st>>>(c.scal + kDotFA, c.scal + kDotGB, c.scal + kAccCol + 2,
                                           static_cast<double>(p->eps), c.ma * c.mb, out);
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return finish(c);
  });
}

size_t fs_solve_host_workspace_bytes(const fs_problem* p) {
  using namespace fs;
  if (!shape_ok(p) || p->d > FS_MAX_D) return 0;
  const size_t n = static_cast<size_t>(p->n), m = static_cast<size_t>(p->m),
               d = static_cast<size_t>(p->d);
  size_t o = fs_workspace_bytes(p);
  o = align_up(o + n * d * 4);      // x
  o = align_up(o + m * d * 4);      // y
  o = align_up(o + n * 4);          // a
  o = align_up(o + m * 4);          // b
  o = align_up(o + n * 4);          // f
  o = align_up(o + m * 4);          // g
  o = align_up(o + n * d * 4);      // grad
  o = align_up(o + 8 * sizeof(double));  // cost + residual
  return o;
}

fs_status fs_solve_host(const fs_problem* hp, int32_t n_iters, float* f, float* g, float* grad_x,
                        double* cost, double* residual, void* ws, size_t ws_bytes,
                        fs_stream_t stream) {
  using namespace fs;
  if (!hp) return FS_ERR_NULL;
  if (!shape_ok(hp)) return FS_ERR_SHAPE;
  if (hp->d > FS_MAX_D) return FS_ERR_UNSUPPORTED_D;
  if (!hp->x || !hp->y || !f || !g) return FS_ERR_NULL;
  if (n_iters < 1) return FS_ERR_ITERS;
  const size_t need = fs_solve_host_workspace_bytes(hp);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 || ws_bytes < need)
    return FS_ERR_WORKSPACE;
  const size_t n = static_cast<size_t>(hp->n), m = static_cast<size_t>(hp->m),
               d = static_cast<size_t>(hp->d);
  const size_t inner = fs_workspace_bytes(hp);
  unsigned char* base = static_cast<unsigned char*>(ws);
  size_t o = inner;
  float* dx = reinterpret_cast<float*>(base + o);
  o = align_up(o + n * d * 4);
  float* dy = reinterpret_cast<float*>(base + o);
  o = align_up(o + m * d * 4);
  float* da = reinterpret_cast<float*>(base + o);
  o = align_up(o + n * 4);
  float* db = reinterpret_cast<float*>(base + o);
  o = align_up(o + m * 4);
  float* df = reinterpret_cast<float*>(base + o);
  o = align_up(o + n * 4);
  float* dg = reinterpret_cast<float*>(base + o);
  o = align_up(o + m * 4);
  float* dgrad = reinterpret_cast<float*>(base + o);
  o = align_up(o + n * d * 4);
  double* dsc = reinterpret_cast<double*>(base + o);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  try {
    CK(cudaMemcpyAsync(dx, hp->x, n * d * 4, cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(dy, hp->y, m * d * 4, cudaMemcpyHostToDevice, st));
    if (hp->a) CK(cudaMemcpyAsync(da, hp->a, n * 4, cudaMemcpyHostToDevice, st));
    if (hp->b) CK(cudaMemcpyAsync(db, hp->b, m * 4, cudaMemcpyHostToDevice, st));
  } catch (const CudaFail&) {
    cudaStreamSynchronize(st);
    cudaGetLastError();
    return FS_ERR_CUDA;
  }
  fs_problem dp = *hp;
  dp.x = dx;
  dp.y = dy;
  dp.a = hp->a ? da : nullptr;
  dp.b = hp->b ? db : nullptr;
  fs_status s = fs_potentials(&dp, n_iters, nullptr, df, dg, ws, inner, stream);
  if (s != FS_OK) return s;
  if (grad_x) {
    s = fs_grad_x(&dp, dg, dgrad, ws, inner, stream);
    if (s != FS_OK) return s;
  }
  if (residual) {
    s = fs_marginal_residual(&dp, df, dg, dsc + 1, nullptr, nullptr, ws, inner, stream);
    if (s != FS_OK) return s;
  }
  if (cost) {
    s = fs_cost(&dp, df, dg, dsc, ws, inner, stream);
    if (s != FS_OK) return s;
  }
  try {
    CK(cudaMemcpyAsync(f, df, n * 4, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(g, dg, m * 4, cudaMemcpyDeviceToHost, st));
    if (grad_x) CK(cudaMemcpyAsync(grad_x, dgrad, n * d * 4, cudaMemcpyDeviceToHost, st));
    if (residual) CK(cudaMemcpyAsync(residual, dsc + 1, 4 * sizeof(double), cudaMemcpyDeviceToHost, st));
    if (cost) CK(cudaMemcpyAsync(cost, dsc, sizeof(double), cudaMemcpyDeviceToHost, st));
    CK(cudaStreamSynchronize(st));
  } catch (const CudaFail&) {
    cudaStreamSynchronize(st);
    cudaGetLastError();
    return FS_ERR_CUDA;
  }
  return FS_OK;
}

int64_t fs_launch_count(void) { return fs::g_launches.load(std::memory_order_relaxed); }

void fs_screening_enable(int on) { fs::g_screening.store(on != 0); }

fs_status fs_workspace_invalidate(void* ws, size_t ws_bytes, fs_stream_t stream) {
  using namespace fs;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 ||
      ws_bytes < kScalarDoubles * sizeof(double))
    return FS_ERR_WORKSPACE;
  // the scalar block opens every layout; the record's first word is its marker
  double* scal = static_cast<double*>(ws);
  try {
    CK(cudaMemsetAsync(scal + kSortMemo, 0, sizeof(unsigned long long),
                       static_cast<cudaStream_t>(stream)));
  } catch (const CudaFail&) {
    return FS_ERR_CUDA;
  }
  return FS_OK;
}

void fs_inject_error_word(unsigned bits) { fs::g_inject.store(bits); }

fs_status fs_check_bounded_wait(int64_t limit_ns, void* ws, size_t ws_bytes, fs_stream_t stream) {
  using namespace fs;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 ||
      ws_bytes < kScalarDoubles * sizeof(double))
    return FS_ERR_WORKSPACE;
  if (limit_ns < 1000 || limit_ns > static_cast<int64_t>(kWaitLimitNs)) return FS_ERR_OPTION;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* err = err_ptr(static_cast<double*>(ws));
  return guarded(st, [&]() -> fs_status {
    CK(cudaMemsetAsync(err, 0, sizeof(unsigned), st));
    bounded_wait_check_kernel<<<1, 32, 0, st>>>(err, static_cast<unsigned long long>(limit_ns));
    CK(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    unsigned h = 0;
    CK(cudaMemcpyAsync(&h, err, sizeof(h), cudaMemcpyDeviceToHost, st));
    CK(cudaStreamSynchronize(st));
    return h ? FS_ERR_TIMEOUT : FS_OK;
  });
}

void fs_timing_enable(int on) {
  std::lock_guard<std::mutex> lk(fs::g_timing_mu);
  fs::g_timing_on = on != 0;
}

void fs_timing_reset(void) {
  std::lock_guard<std::mutex> lk(fs::g_timing_mu);
  fs::g_timing = fs_timing{};
}

void fs_timing_get(fs_timing* out) {
  if (!out) return;
  std::lock_guard<std::mutex> lk(fs::g_timing_mu);
  *out = fs::g_timing;
}

}  // extern "C"
