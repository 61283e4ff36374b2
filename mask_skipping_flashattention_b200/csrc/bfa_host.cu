// Host side of the C ABI declared in include/bfa.h: argument validation, plan
// allocation and layout, TMA tensor maps, and the kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/bfa.h"
#include "bwd_params.cuh"
#include "fwd_params.cuh"
#include "plan_types.cuh"

#define BFA_API extern "C" __attribute__((visibility("default")))

namespace bfa {

// kernels (planner.cu, fwd.cu)
// With `groups` set, the launch also writes the dense plan's single group
// (*group), its row -> group map and clears the status words.
cudaError_t launch_dense_classify(const uint8_t* mask, int64_t ld, int Sq, int Sk, uint8_t* cls, uint32_t* fine,
                                  cudaStream_t s, GroupInfo* groups = nullptr, const GroupInfo* group = nullptr,
                                  int32_t* row_group = nullptr, uint32_t* err = nullptr, int32_t* max_width = nullptr);
cudaError_t launch_blockid_classify(const GroupInfo* groups, int n_groups, int max_tiles_q, int max_tiles_k,
                                    const int32_t* q_blk, const int32_t* k_blk, const uint8_t* q_valid,
                                    const uint8_t* k_valid, int batched, int Sq, int Sk, int window, int copy_ids,
                                    int32_t* qid, uint8_t* qv, int32_t* kid, uint32_t* kbits, uint8_t* cls,
                                    cudaStream_t s);
cudaError_t launch_bsr_classify(const int32_t* indptr, const int32_t* indices, int64_t n_indices,
                                const GroupInfo* groups, int n_groups, int nqt, int causal, uint8_t* cls,
                                uint32_t* err, int32_t* max_width, cudaStream_t s);
cudaError_t launch_rows(const GroupInfo* groups, const int32_t* row_group, const uint8_t* cls, int n_rows,
                        int max_nkt, int32_t* row_cnt, int32_t* row_ptr, int32_t* kv_tile, int32_t* part,
                        int32_t* order, cudaStream_t s, int32_t* pair_row = nullptr, int32_t* pair_cost = nullptr,
                        int32_t* pair_order = nullptr, int32_t* pair_idx = nullptr, int part_is_pos = 0,
                        int2* row_work = nullptr, int2* pair_work = nullptr, int n_groups = 0,
                        int64_t grid_tiles = -1);
cudaError_t launch_bsr_to_bits(const int32_t* indptr, const int32_t* indices, int64_t n_indices, int n_groups,
                               int nqb, int nkb, int wpr, uint32_t* bits, uint32_t* err, cudaStream_t s);
cudaError_t launch_cols(const GroupInfo* groups, int n_groups, const uint8_t* cls, const int32_t* row_ptr,
                        const int32_t* kv_tile, int part_is_pos, int max_nqt, int n_cols, int32_t* col0,
                        int32_t* col_group, int32_t* col_cnt, int32_t* col_ptr, int32_t* q_tile, int32_t* tpart,
                        int32_t* col_order, cudaStream_t s);
cudaError_t launch_bits_classify(const uint32_t* bits, const uint32_t* kv_valid, int nqb, int wpr, int kv_wpb,
                                 int q_block, int kv_block, int causal, int g_pack, const GroupInfo* groups,
                                 int n_groups, int nqt, uint8_t* cls, cudaStream_t s);
cudaError_t launch_bits_fine(const uint32_t* bits, const uint32_t* kv_valid, int nqb, int wpr, int kv_wpb,
                             int q_block, int kv_block, int causal, int g_pack, const GroupInfo* groups,
                             const int32_t* row_group, int n_rows, const int32_t* row_ptr, const int32_t* kv_tile,
                             const int32_t* part, uint32_t* fine, cudaStream_t s);
cudaError_t launch_make_block_ids(const uint8_t* pad, const uint8_t* att, int B, int N, int n_cross,
                                  const uint8_t* cross_pad, int32_t* q_blk, int32_t* k_blk, uint8_t* q_valid,
                                  uint8_t* k_valid, cudaStream_t s);
cudaError_t launch_pred_classify(const int32_t* terms, int n_terms, const GroupInfo* groups, int n_groups, int nqt,
                                 uint8_t* cls, cudaStream_t s);
cudaError_t launch_init_regular_groups(const GroupInfo& tmpl, int n_groups, int n_hkv, int bsr, int copy_ids,
                                       GroupInfo* groups, int32_t* row_group, int n_rows, cudaStream_t s,
                                       uint32_t* err = nullptr, int32_t* max_width = nullptr);
cudaError_t launch_check_guards(const void* slab, const uint64_t* offs, int n, uint32_t guard_bytes, int guard_byte,
                                uint32_t* err, cudaStream_t s);


}  // namespace bfa

using namespace bfa;

// ----------------------------------------------------------------------------
// plan object
// ----------------------------------------------------------------------------
struct bfa_plan {
  int kind = 0, varlen = 0, batch = 0, hkv = 0, sq = 0, sk = 0, window = -1, causal = 0;
  // GQA-packed query rows (bfa_plan_bsr_packed): plan row t of a (batch, kv head)
  // group is query position t / pack_g of head t % pack_g of the kv head; 1: off
  int pack_g = 1;
  int n_groups = 0, n_rows = 0, n_pairs = 0, max_nkt = 0, max_nqt = 0, mask_mode = MASK_BITS;
  int64_t grid_tiles = 0;
  int64_t fine_tiles = 0;       // tiles of packed fine words held in `fine`
  void* fine_extra = nullptr;   // separately allocated fine words (generic block sparsity)
  bool regular = false;   // every group the same shape: the group table is built on the device
  int regular_hkv = 1;    // groups per batch of a regular layout (BSR: Hkv)
  bool copy_ids = false;
  std::vector<GroupInfo> groups_h;
  cudaStream_t stream = nullptr;
  void* slab = nullptr;
  // device arrays inside the slab
  GroupInfo* groups = nullptr;
  int32_t* row_group = nullptr;
  uint8_t* cls = nullptr;
  int32_t* row_cnt = nullptr;
  int32_t* row_ptr = nullptr;
  int32_t* kv_tile = nullptr;
  int32_t* part = nullptr;
  uint32_t* fine = nullptr;
  int32_t* order = nullptr;
  int32_t* pair_row = nullptr;    // first row of each work pair (~row: single-row pair)
  int32_t* pair_cost = nullptr;   // listed tiles of the pair
  int32_t* pair_order = nullptr;  // longest-first order of the pairs
  int32_t* pair_idx = nullptr;    // scratch: pair index of each row
  int2* row_work = nullptr;       // rows in longest-first order with their group
  int2* pair_work = nullptr;      // pairs in longest-first order with the group of their first row
  int32_t* qid = nullptr;
  uint8_t* qvalid = nullptr;
  int32_t* kid = nullptr;
  uint32_t* kbits = nullptr;
  int32_t* terms = nullptr;
  int n_terms = 0;
  uint32_t* err = nullptr;
  int32_t* max_width = nullptr;
  int part_is_pos = 0;    // partial entries index the fine words by list position (else by grid index)
  // transposed lists (built on first use by the backward or an export)
  void* cols_slab = nullptr;
  int32_t* col0 = nullptr;       // [n_groups + 1] first column of each group
  int32_t* col_group = nullptr;  // [n_cols]
  int32_t* col_cnt = nullptr;    // [n_cols]
  int32_t* col_ptr = nullptr;    // [n_cols + 1]
  int32_t* q_tile = nullptr;     // [listed tiles]
  int32_t* tpart = nullptr;      // [listed tiles]
  int32_t* col_order = nullptr;  // [n_cols]
  // capacities of the id copies (entries), for the checked build's index checks
  int64_t cap_qid = 1, cap_kid = 1, cap_kbits = 1;
  // checked build: guard regions after every slab array (offsets into the slab,
  // held in the slab's last region so that a kernel can verify them)
  int n_guards = 0, n_col_guards = 0;
  const uint64_t* guard_offs = nullptr;
  const uint64_t* col_guard_offs = nullptr;
  std::vector<uint64_t> guards_h, col_guards_h;
};

namespace {

thread_local std::string g_err;
uint64_t g_wait_ns = 1000000000ull;
int g_bwd_deterministic = 0;  // bfa_set_bwd_deterministic

// Device address of the allocation-free planner's scratch array, per device
// (looked up on that entry point's first call on a device; see below).
std::mutex g_noalloc_mu;
uint8_t* g_noalloc_ptr[64] = {};

bfa_status fail(bfa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

bfa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(BFA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define BFA_CUDA(call, what)                  \
  do {                                        \
    cudaError_t e_ = (call);                  \
    if (e_ != cudaSuccess) {                  \
      cleanup();                              \
      return cuda_fail(e_, what);             \
    }                                         \
  } while (0)

// BFA_ERR_NOT_DEVICE unless p is device (or managed) memory.
bfa_status need_device(const void* p, const char* name, bool allow_null = false) {
  if (p == nullptr) {
    if (allow_null) return BFA_OK;
    return fail(BFA_ERR_INVALID_ARG, "%s is NULL", name);
  }
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(BFA_ERR_NOT_DEVICE, "%s is not a device pointer (%s)", name, cudaGetErrorString(e));
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return fail(BFA_ERR_NOT_DEVICE, "%s is not device memory (CPU tensors are not supported)", name);
  return BFA_OK;
}

// Stream-ordered pool for plan memory, one per device.  Its release threshold
// is unbounded, so building and freeing plans in a loop reuses the same memory
// instead of returning it to the driver at every synchronisation.
cudaError_t plan_pool(cudaMemPool_t* out) {
  static cudaMemPool_t pools[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!pools[dev]) {
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool;
    e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) return e;
    uint64_t thr = UINT64_MAX;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &thr);
    if (e != cudaSuccess) return e;
    pools[dev] = pool;
  }
  *out = pools[dev];
  return cudaSuccess;
}

constexpr int kMaxKvTiles = 16384;  // key tiles per row: the row kernel's shared-memory buckets

inline int cdiv(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// The checked build places kGuardBytes of guard bytes (kGuardByte) right after
// every array of a slab; bfa_plan_device_status verifies them.
constexpr size_t kGuardBytes = 64;
constexpr int kGuardByte = 0xA5;
#ifdef BFA_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif

struct SlabLayout {
  size_t off = 0;
  std::vector<uint64_t> guards;  // checked build: offsets of the guard regions
  template <typename T>
  size_t take(size_t count) {
    const size_t o = off;
    const size_t end = off + count * sizeof(T);
    if (kChecked) {
      guards.push_back(end);
      off = align256(end + kGuardBytes);
    } else {
      off = align256(end);
    }
    return o;
  }
  // checked build: room for the guard offsets at the end of the slab
  size_t take_guard_table() { return take<uint64_t>(guards.size() + 1); }
};

// checked build: fill a new slab with the guard byte and upload its guard table
cudaError_t arm_guards(void* slab, size_t bytes, SlabLayout& L, size_t o_table, std::vector<uint64_t>& keep,
                       cudaStream_t st) {
  if (!kChecked) return cudaSuccess;
  keep = L.guards;
  keep.pop_back();  // the table's own guard is not listed (it is written by the upload)
  cudaError_t e = cudaMemsetAsync(slab, kGuardByte, bytes, st);
  if (e == cudaSuccess && !keep.empty())
    e = cudaMemcpyAsync(static_cast<uint8_t*>(slab) + o_table, keep.data(), keep.size() * sizeof(uint64_t),
                        cudaMemcpyHostToDevice, st);
  return e;
}

// Allocate and carve the plan slab; uploads groups and row_group.
// `init_later`: a regular layout whose group table and status words the
// caller's first kernel writes (dense plans: the classify launch).
bfa_status alloc_plan(bfa_plan* P, bool with_fine, int64_t qid_elems, int64_t kid_elems, int64_t kbit_words,
                      int64_t term_ints = 0, bool init_later = false) {
  SlabLayout L;
  const int64_t cap_tiles = std::max<int64_t>(P->grid_tiles, 1);
  const size_t o_groups = L.take<GroupInfo>(std::max(P->n_groups, 1));
  const size_t o_rowg = L.take<int32_t>(std::max(P->n_rows, 1));
  const size_t o_cls = L.take<uint8_t>(cap_tiles);
  const size_t o_cnt = L.take<int32_t>(std::max(P->n_rows, 1));
  const size_t o_ptr = L.take<int32_t>(P->n_rows + 1);
  const size_t o_kv = L.take<int32_t>(cap_tiles);
  const size_t o_part = L.take<int32_t>(cap_tiles);
  const size_t o_ord = L.take<int32_t>(std::max(P->n_rows, 1));
  const size_t o_prow = L.take<int32_t>(std::max(P->n_rows, 1));
  const size_t o_pcost = L.take<int32_t>(std::max(P->n_rows, 1));
  const size_t o_pord = L.take<int32_t>(std::max(P->n_rows, 1));
  const size_t o_pidx = L.take<int32_t>(std::max(P->n_rows, 1));
  const size_t o_rwork = L.take<int2>(std::max(P->n_rows, 1));
  const size_t o_pwork = L.take<int2>(std::max(P->n_rows, 1));
  const size_t o_err = L.take<uint32_t>(1);
  const size_t o_mw = L.take<int32_t>(1);
  const size_t o_qid = L.take<int32_t>(std::max<int64_t>(qid_elems, 1));
  const size_t o_qv = L.take<uint8_t>(std::max<int64_t>(qid_elems, 1));
  const size_t o_kid = L.take<int32_t>(std::max<int64_t>(kid_elems, 1));
  const size_t o_kb = L.take<uint32_t>(std::max<int64_t>(kbit_words, 1));
  const size_t o_terms = L.take<int32_t>(std::max<int64_t>(term_ints, 1));
  const size_t o_fine = L.take<uint32_t>(with_fine ? static_cast<size_t>(cap_tiles) * kFineWordsPerTile : 1);
  const size_t o_gtab = kChecked ? L.take_guard_table() : 0;
  P->cap_qid = std::max<int64_t>(qid_elems, 1);
  P->cap_kid = std::max<int64_t>(kid_elems, 1);
  P->cap_kbits = std::max<int64_t>(kbit_words, 1);
  cudaMemPool_t pool;
  cudaError_t e = plan_pool(&pool);
  if (e != cudaSuccess) return cuda_fail(e, "plan memory pool");
  e = cudaMallocFromPoolAsync(&P->slab, L.off, pool, P->stream);
  if (e != cudaSuccess) return fail(BFA_ERR_CAPACITY, "plan allocation of %zu bytes failed: %s", L.off,
                                    cudaGetErrorString(e));
  uint8_t* base = static_cast<uint8_t*>(P->slab);
  e = arm_guards(P->slab, L.off, L, o_gtab, P->guards_h, P->stream);
  if (e != cudaSuccess) return cuda_fail(e, "plan guard bytes");
  P->n_guards = static_cast<int>(P->guards_h.size());
  P->guard_offs = reinterpret_cast<const uint64_t*>(base + o_gtab);
  P->groups = reinterpret_cast<GroupInfo*>(base + o_groups);
  P->row_group = reinterpret_cast<int32_t*>(base + o_rowg);
  P->cls = base + o_cls;
  P->row_cnt = reinterpret_cast<int32_t*>(base + o_cnt);
  P->row_ptr = reinterpret_cast<int32_t*>(base + o_ptr);
  P->kv_tile = reinterpret_cast<int32_t*>(base + o_kv);
  P->part = reinterpret_cast<int32_t*>(base + o_part);
  P->order = reinterpret_cast<int32_t*>(base + o_ord);
  P->pair_row = reinterpret_cast<int32_t*>(base + o_prow);
  P->pair_cost = reinterpret_cast<int32_t*>(base + o_pcost);
  P->pair_order = reinterpret_cast<int32_t*>(base + o_pord);
  P->pair_idx = reinterpret_cast<int32_t*>(base + o_pidx);
  P->row_work = reinterpret_cast<int2*>(base + o_rwork);
  P->pair_work = reinterpret_cast<int2*>(base + o_pwork);
  P->err = reinterpret_cast<uint32_t*>(base + o_err);
  P->max_width = reinterpret_cast<int32_t*>(base + o_mw);
  P->qid = reinterpret_cast<int32_t*>(base + o_qid);
  P->qvalid = base + o_qv;
  P->kid = reinterpret_cast<int32_t*>(base + o_kid);
  P->kbits = reinterpret_cast<uint32_t*>(base + o_kb);
  P->terms = reinterpret_cast<int32_t*>(base + o_terms);
  P->fine = reinterpret_cast<uint32_t*>(base + o_fine);

  if (P->regular && init_later) {
    // nothing to launch here
  } else if (P->regular) {
    // the same launch clears the status words (err, max_width)
    e = launch_init_regular_groups(P->groups_h[0], P->n_groups, P->regular_hkv, P->kind == BFA_PLAN_BSR ? 1 : 0,
                                   P->copy_ids ? 1 : 0, P->groups, P->row_group, P->n_rows, P->stream, P->err,
                                   P->max_width);
    if (e != cudaSuccess) return cuda_fail(e, "plan group table kernel");
  } else {
    // irregular (varlen) layouts: the planner has synchronised already to read
    // the sequence lengths, so a pageable upload costs nothing extra here
    std::vector<int32_t> rg(std::max(P->n_rows, 1), 0);
    for (int g = 0; g < P->n_groups; ++g)
      for (int r = 0; r < P->groups_h[g].nqt; ++r) rg[P->groups_h[g].row0 + r] = g;
    if (P->n_groups > 0) {
      e = cudaMemcpyAsync(P->groups, P->groups_h.data(), sizeof(GroupInfo) * P->n_groups, cudaMemcpyHostToDevice,
                          P->stream);
      if (e != cudaSuccess) return cuda_fail(e, "upload plan groups");
    }
    e = cudaMemcpyAsync(P->row_group, rg.data(), sizeof(int32_t) * rg.size(), cudaMemcpyHostToDevice, P->stream);
    if (e != cudaSuccess) return cuda_fail(e, "upload plan rows");
  }
  if (!P->regular) {  // regular layouts cleared them in the group-table launch
    e = cudaMemsetAsync(P->err, 0, sizeof(uint32_t), P->stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(P->max_width, 0, sizeof(int32_t), P->stream);
    if (e != cudaSuccess) return cuda_fail(e, "clear plan status");
  }
  return BFA_OK;
}

void free_plan(bfa_plan* P) {
  if (!P) return;
  if (P->cols_slab) cudaFreeAsync(P->cols_slab, P->stream);
  if (P->fine_extra) cudaFreeAsync(P->fine_extra, P->stream);
  if (P->slab) cudaFreeAsync(P->slab, P->stream);
  delete P;
}

// Finish the plan: groups laid out, classes written -> lists and order.
bfa_status build_rows(bfa_plan* P, int part_is_pos = 0) {
  P->part_is_pos = part_is_pos;
  if (P->n_rows == 0) {
    cudaError_t e = cudaMemsetAsync(P->row_ptr, 0, sizeof(int32_t), P->stream);
    return e == cudaSuccess ? BFA_OK : cuda_fail(e, "empty plan");
  }
  if (P->max_nkt > kMaxKvTiles) return fail(BFA_ERR_CAPACITY, "too many key tiles per row (%d)", P->max_nkt);
  cudaError_t e = launch_rows(P->groups, P->row_group, P->cls, P->n_rows, P->max_nkt, P->row_cnt, P->row_ptr,
                              P->kv_tile, P->part, P->order, P->stream, P->pair_row, P->pair_cost,
                              P->pair_order, P->pair_idx, part_is_pos, P->row_work, P->pair_work, P->n_groups,
                              P->grid_tiles);
  return e == cudaSuccess ? BFA_OK : cuda_fail(e, "plan rows kernel");
}

// Key-tile columns of the plan: every group's key tiles, groups in order.
int plan_n_cols(const bfa_plan* P) {
  if (P->regular) return P->groups_h.empty() ? 0 : P->n_groups * P->groups_h[0].nkt;
  int n = 0;
  for (const auto& g : P->groups_h) n += g.nkt;
  return n;
}

// Build the transposed lists on `st` unless they exist.
bfa_status ensure_cols(bfa_plan* P, cudaStream_t st) {
  if (P->cols_slab) return BFA_OK;
  const int n_cols = plan_n_cols(P);
  SlabLayout L;
  const int64_t cap = std::max<int64_t>(P->grid_tiles, 1);
  const size_t o_c0 = L.take<int32_t>(P->n_groups + 1);
  const size_t o_cg = L.take<int32_t>(std::max(n_cols, 1));
  const size_t o_cc = L.take<int32_t>(std::max(n_cols, 1));
  const size_t o_cp = L.take<int32_t>(n_cols + 1);
  const size_t o_qt = L.take<int32_t>(cap);
  const size_t o_tp = L.take<int32_t>(cap);
  const size_t o_co = L.take<int32_t>(std::max(n_cols, 1));
  const size_t o_gtab = kChecked ? L.take_guard_table() : 0;
  cudaMemPool_t pool;
  cudaError_t e = plan_pool(&pool);
  if (e != cudaSuccess) return cuda_fail(e, "plan memory pool");
  e = cudaMallocFromPoolAsync(&P->cols_slab, L.off, pool, st);
  if (e != cudaSuccess) {
    P->cols_slab = nullptr;
    return fail(BFA_ERR_CAPACITY, "transposed plan allocation of %zu bytes failed: %s", L.off, cudaGetErrorString(e));
  }
  uint8_t* base = static_cast<uint8_t*>(P->cols_slab);
  e = arm_guards(P->cols_slab, L.off, L, o_gtab, P->col_guards_h, st);
  if (e != cudaSuccess) return cuda_fail(e, "transposed plan guard bytes");
  P->n_col_guards = static_cast<int>(P->col_guards_h.size());
  P->col_guard_offs = reinterpret_cast<const uint64_t*>(base + o_gtab);
  P->col0 = reinterpret_cast<int32_t*>(base + o_c0);
  P->col_group = reinterpret_cast<int32_t*>(base + o_cg);
  P->col_cnt = reinterpret_cast<int32_t*>(base + o_cc);
  P->col_ptr = reinterpret_cast<int32_t*>(base + o_cp);
  P->q_tile = reinterpret_cast<int32_t*>(base + o_qt);
  P->tpart = reinterpret_cast<int32_t*>(base + o_tp);
  P->col_order = reinterpret_cast<int32_t*>(base + o_co);
  if (n_cols == 0 || P->n_groups == 0) {
    e = cudaMemsetAsync(P->col_ptr, 0, sizeof(int32_t), st);
    return e == cudaSuccess ? BFA_OK : cuda_fail(e, "empty transposed plan");
  }
  if (P->max_nqt > kMaxKvTiles) return fail(BFA_ERR_CAPACITY, "too many query tiles per column (%d)", P->max_nqt);
  e = launch_cols(P->groups, P->n_groups, P->cls, P->row_ptr, P->kv_tile, P->part_is_pos, std::max(P->max_nqt, 1),
                  n_cols, P->col0, P->col_group, P->col_cnt, P->col_ptr, P->q_tile, P->tpart, P->col_order, st);
  return e == cudaSuccess ? BFA_OK : cuda_fail(e, "transposed plan kernel");
}

void finalize_layout(bfa_plan* P) {
  int row = 0;
  int64_t cls = 0;
  P->max_nkt = 0;
  P->max_nqt = 0;
  P->n_pairs = 0;
  for (auto& g : P->groups_h) {
    g.row0 = row;
    g.cls_off = cls;
    row += g.nqt;
    P->n_pairs += (g.nqt + 1) / 2;
    cls += static_cast<int64_t>(g.nqt) * g.nkt;
    P->max_nkt = std::max(P->max_nkt, g.nkt);
    P->max_nqt = std::max(P->max_nqt, g.nqt);
  }
  P->n_rows = row;
  P->grid_tiles = cls;
  P->n_groups = static_cast<int>(P->groups_h.size());
}

GroupInfo make_group(int q_off, int q_len, int k_off, int k_len, int b, int hkv) {
  GroupInfo g;
  std::memset(&g, 0, sizeof(g));
  g.q_off = q_off;
  g.q_len = q_len;
  g.k_off = k_off;
  g.k_len = k_len;
  g.b = b;
  g.hkv = hkv;
  g.nqt = cdiv(q_len, kTile);
  g.nkt = cdiv(k_len, kTile);
  return g;
}

bfa_status check_capacity(const bfa_plan* P, bool with_fine) {
  if (P->grid_tiles >= (int64_t(1) << 31)) return fail(BFA_ERR_CAPACITY, "class grid of %lld tiles exceeds int32",
                                                       (long long)P->grid_tiles);
  if (with_fine && P->grid_tiles * 2048 > (int64_t(64) << 30))
    return fail(BFA_ERR_CAPACITY, "fine-mask capacity %lld bytes too large", (long long)(P->grid_tiles * 2048));
  return BFA_OK;
}

}  // namespace

// ----------------------------------------------------------------------------
// C ABI
// ----------------------------------------------------------------------------
BFA_API const char* bfa_version(void) { return kChecked ? "bfa 0.1 (sm_100a, checked)" : "bfa 0.1 (sm_100a)"; }

BFA_API const char* bfa_last_error(void) { return g_err.c_str(); }

BFA_API int bfa_is_available(void) {
  int n = 0;
  cudaError_t e = cudaGetDeviceCount(&n);
  if (e != cudaSuccess || n == 0) {
    cudaGetLastError();
    fail(BFA_ERR_CUDA, "no CUDA device: %s", e == cudaSuccess ? "count is 0" : cudaGetErrorString(e));
    return 0;
  }
  int dev = 0, major = 0, minor = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) {
    fail(BFA_ERR_UNSUPPORTED, "device is sm_%d%d; these kernels are built for sm_100a only", major, minor);
    return 0;
  }
  e = probe_fwd_kernels();
  if (e != cudaSuccess) {
    fail(BFA_ERR_CUDA, "kernel image does not load: %s", cudaGetErrorString(e));
    return 0;
  }
  // A device reset reloads the library's device code, and the scratch array of
  // the allocation-free planner may then sit at another address: forget the one
  // looked up before, so that planner's next call on this device looks it up again.
  if (dev >= 0 && dev < 64) {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    g_noalloc_ptr[dev] = nullptr;
  }
  return 1;
}

BFA_API void bfa_set_wait_timeout_ns(uint64_t ns) {
  if (ns == 0) ns = 1000000000ull;
  g_wait_ns = std::min<uint64_t>(std::max<uint64_t>(ns, BFA_WAIT_NS_MIN), BFA_WAIT_NS_MAX);
}

BFA_API void bfa_set_bwd_deterministic(int on) { g_bwd_deterministic = on ? 1 : 0; }

BFA_API bfa_status bfa_make_block_ids(const uint8_t* pad_masks, const uint8_t* att_masks, int B, int N, int n_cross,
                                      const uint8_t* cross_pad, int32_t* q_blk, int32_t* k_blk, uint8_t* q_valid,
                                      uint8_t* k_valid, void* stream) {
  if (B <= 0 || N <= 0 || n_cross < 0) return fail(BFA_ERR_INVALID_ARG, "bad sizes B=%d N=%d n_cross=%d", B, N, n_cross);
  bfa_status s;
  if ((s = need_device(pad_masks, "pad_masks")) || (s = need_device(att_masks, "att_masks")) ||
      (s = need_device(q_blk, "q_blk")) || (s = need_device(k_blk, "k_blk")) ||
      (s = need_device(q_valid, "q_valid")) || (s = need_device(k_valid, "k_valid")))
    return s;
  if (n_cross > 0 && (s = need_device(cross_pad, "cross_pad"))) return s;
  cudaError_t e = launch_make_block_ids(pad_masks, att_masks, B, N, n_cross, cross_pad, q_blk, k_blk, q_valid,
                                        k_valid, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? BFA_OK : cuda_fail(e, "make_block_ids kernel");
}

BFA_API bfa_status bfa_plan_dense(const uint8_t* mask, int64_t ld, int Sq, int Sk, bfa_plan** out, void* stream) {
  if (!out) return fail(BFA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (Sq <= 0 || Sk <= 0) return fail(BFA_ERR_INVALID_ARG, "Sq=%d Sk=%d must be positive", Sq, Sk);
  if (ld < Sk) return fail(BFA_ERR_INVALID_ARG, "mask_row_stride %lld < Sk %d", (long long)ld, Sk);
  bfa_status s = need_device(mask, "mask");
  if (s) return s;
  bfa_plan* P = new bfa_plan();
  auto cleanup = [&]() { free_plan(P); };
  P->kind = BFA_PLAN_DENSE;
  P->stream = static_cast<cudaStream_t>(stream);
  P->sq = Sq;
  P->sk = Sk;
  P->mask_mode = MASK_BITS;
  P->groups_h.push_back(make_group(0, Sq, 0, Sk, -1, -1));
  P->regular = true;
  finalize_layout(P);
  if ((s = check_capacity(P, true))) { cleanup(); return s; }
  if ((s = alloc_plan(P, true, 0, 0, 0, 0, /*init_later=*/true))) { cleanup(); return s; }
  P->fine_tiles = P->grid_tiles;
  GroupInfo g0 = P->groups_h[0];
  BFA_CUDA(launch_dense_classify(mask, ld, Sq, Sk, P->cls, P->fine, P->stream, P->groups, &g0, P->row_group, P->err,
                                 P->max_width),
           "dense classify kernel");
  if ((s = build_rows(P))) { cleanup(); return s; }
  *out = P;
  return BFA_OK;
}

namespace {

// Row groups of a batched (B x Sq x Sk) or varlen (cu_seqlens) layout, with the
// usable keys optionally bounded by seqused_k.  Varlen lengths and seqused_k are
// read back to the host (one synchronisation) and validated against max_q / max_k.
bfa_status setup_seq_groups(bfa_plan* P, int B, int Sq, int Sk, const int32_t* cu_q, const int32_t* cu_k,
                            const int32_t* seqused_k, int max_q, int max_k, cudaStream_t st) {
  auto cleanup = []() {};
  const bool varlen = cu_q != nullptr;
  if (varlen) {
    std::vector<int32_t> cq(B + 1), ck(B + 1);
    BFA_CUDA(cudaMemcpyAsync(cq.data(), cu_q, sizeof(int32_t) * (B + 1), cudaMemcpyDeviceToHost, st), "read cu_seqlens_q");
    BFA_CUDA(cudaMemcpyAsync(ck.data(), cu_k, sizeof(int32_t) * (B + 1), cudaMemcpyDeviceToHost, st), "read cu_seqlens_k");
    BFA_CUDA(cudaStreamSynchronize(st), "read cu_seqlens");
    if (cq[0] != 0 || ck[0] != 0) { return fail(BFA_ERR_INVALID_ARG, "cu_seqlens must start at 0"); }
    for (int i = 0; i < B; ++i) {
      const int lq = cq[i + 1] - cq[i], lk = ck[i + 1] - ck[i];
      if (lq < 0 || lk < 0) { return fail(BFA_ERR_INVALID_ARG, "cu_seqlens decreases at sequence %d", i); }
      if (lq > max_q || lk > max_k) {
        return fail(BFA_ERR_INVALID_ARG, "sequence %d has lengths (%d, %d) above max_q=%d / max_k=%d", i, lq, lk,
                    max_q, max_k);
      }
      P->groups_h.push_back(make_group(cq[i], lq, ck[i], lk, 0, -1));
    }
    P->sq = cq[B];
    P->sk = ck[B];
  } else {
    if (Sq <= 0 || Sk <= 0) { return fail(BFA_ERR_INVALID_ARG, "Sq=%d Sk=%d must be positive", Sq, Sk); }
    for (int b = 0; b < B; ++b) P->groups_h.push_back(make_group(0, Sq, 0, Sk, b, -1));
    P->sq = Sq;
    P->sk = Sk;
  }
  P->regular = !varlen;
  if (seqused_k) {  // usable keys per batch entry / sequence (read back once)
    std::vector<int32_t> used(B);
    BFA_CUDA(cudaMemcpyAsync(used.data(), seqused_k, sizeof(int32_t) * B, cudaMemcpyDeviceToHost, st), "read seqused_k");
    BFA_CUDA(cudaStreamSynchronize(st), "read seqused_k");
    for (int b = 0; b < B; ++b) {
      GroupInfo& g = P->groups_h[b];
      if (used[b] < 0) { return fail(BFA_ERR_INVALID_ARG, "seqused_k[%d] = %d is negative", b, used[b]); }
      g.k_len = std::min(g.k_len, used[b]);
      g.nkt = cdiv(g.k_len, kTile);
    }
    P->regular = false;
  }
  return BFA_OK;
}

}  // namespace

BFA_API bfa_status bfa_plan_blockids(const int32_t* q_blk, const int32_t* k_blk, const uint8_t* q_valid,
                                     const uint8_t* k_valid, int B, int Sq, int Sk, const int32_t* cu_q,
                                     const int32_t* cu_k, const int32_t* seqused_k, int max_q, int max_k,
                                     int window_left, bfa_plan** out, void* stream) {
  if (!out) return fail(BFA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (B <= 0) return fail(BFA_ERR_INVALID_ARG, "B=%d must be positive", B);
  if ((q_blk == nullptr) != (k_blk == nullptr))
    return fail(BFA_ERR_INVALID_ARG, "q_blk and k_blk must both be given or both be NULL");
  if ((cu_q == nullptr) != (cu_k == nullptr))
    return fail(BFA_ERR_INVALID_ARG, "cu_seqlens_q and cu_seqlens_k must both be given or both be NULL");
  if (window_left < -1 || window_left == 0) return fail(BFA_ERR_INVALID_ARG, "window_left=%d (use -1 or >= 1)", window_left);
  const bool positional = q_blk == nullptr;
  const bool have_valid = q_valid != nullptr || k_valid != nullptr;
  if (window_left >= 1 && (!positional || have_valid))
    return fail(BFA_ERR_UNSUPPORTED, "a window needs positional ids and no validity masks");
  bfa_status s;
  if ((s = need_device(q_blk, "q_blk", true)) || (s = need_device(k_blk, "k_blk", true)) ||
      (s = need_device(q_valid, "q_valid", true)) || (s = need_device(k_valid, "k_valid", true)) ||
      (s = need_device(cu_q, "cu_seqlens_q", true)) || (s = need_device(cu_k, "cu_seqlens_k", true)) ||
      (s = need_device(seqused_k, "seqused_k", true)))
    return s;
  const bool varlen = cu_q != nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bfa_plan* P = new bfa_plan();
  auto cleanup = [&]() { free_plan(P); };
  P->kind = positional && !have_valid ? BFA_PLAN_POSITIONAL : BFA_PLAN_BLOCKIDS;
  P->mask_mode = positional && !have_valid ? MASK_POS : MASK_BLOCKID;
  P->causal = 1;
  P->window = window_left >= 1 ? window_left : -1;
  P->varlen = varlen;
  P->batch = B;
  P->stream = st;
  if ((s = setup_seq_groups(P, B, Sq, Sk, cu_q, cu_k, seqused_k, max_q, max_k, st))) { cleanup(); return s; }
  P->copy_ids = P->mask_mode == MASK_BLOCKID;
  finalize_layout(P);
  // padded per-group id copies (block-id mode only)
  int64_t qe = 0, ke = 0, kw = 0;
  const bool copy_ids = P->copy_ids;
  for (auto& g : P->groups_h) {
    g.qid_off = static_cast<int32_t>(qe);
    g.kid_off = static_cast<int32_t>(ke);
    g.kbit_off = static_cast<int32_t>(kw);
    if (copy_ids) {
      qe += static_cast<int64_t>(g.nqt) * kTile;
      ke += static_cast<int64_t>(g.nkt) * kTile;
      kw += static_cast<int64_t>(g.nkt) * kWordsPerTileRow;
    }
  }
  if (qe >= (int64_t(1) << 31) || ke >= (int64_t(1) << 31)) { cleanup(); return fail(BFA_ERR_CAPACITY, "too many tokens"); }
  if ((s = check_capacity(P, false))) { cleanup(); return s; }
  if ((s = alloc_plan(P, false, qe, ke, kw))) { cleanup(); return s; }
  if (P->n_groups > 0) {
    BFA_CUDA(launch_blockid_classify(P->groups, P->n_groups, P->max_nqt, P->max_nkt, q_blk, k_blk, q_valid, k_valid,
                                     varlen ? 0 : 1, P->sq, P->sk, P->window, copy_ids ? 1 : 0, P->qid, P->qvalid,
                                     P->kid, P->kbits, P->cls, st),
             "block-id classify kernel");
  }
  if ((s = build_rows(P))) { cleanup(); return s; }
  *out = P;
  return BFA_OK;
}

namespace {

bool kv_block_ok(int kv_block) { return kv_block == 8 || kv_block == 16 || kv_block == 32 || (kv_block > 0 && kv_block % 64 == 0); }

// Block sparsity of any block size (flashinfer block_sparse_attention: BSR rows or
// an exact-block bitmap, key validity bits, dense or causal inside the blocks),
// reduced to tile classes plus packed fine words for the partial tiles.
bfa_status plan_block_sparse(const int32_t* indptr, const int32_t* indices, int64_t n_indices,
                             const uint32_t* block_bits, const uint32_t* kv_valid, int B, int Hkv, int Sq, int Skv,
                             int q_block, int kv_block, int causal, bfa_plan** out, cudaStream_t st,
                             int g_pack = 1) {
  bfa_plan* P = new bfa_plan();
  uint32_t* tmp_bits = nullptr;
  auto cleanup = [&]() {
    if (tmp_bits) cudaFreeAsync(tmp_bits, st);
    free_plan(P);
  };
  bfa_status s;
  P->kind = BFA_PLAN_BSR;
  P->mask_mode = MASK_BITS;
  P->causal = causal ? 1 : 0;
  P->window = -1;
  P->batch = B;
  P->hkv = Hkv;
  P->sq = Sq;
  P->sk = Skv;
  P->stream = st;
  P->pack_g = g_pack;
  // packed: each group's plan rows are its Sq positions x g_pack heads
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) P->groups_h.push_back(make_group(0, Sq * g_pack, 0, Skv, b, h));
  P->regular = true;
  P->regular_hkv = Hkv;
  finalize_layout(P);
  if ((s = check_capacity(P, false))) { cleanup(); return s; }
  if ((s = alloc_plan(P, false, 0, 0, 0))) { cleanup(); return s; }
  const int nqb = cdiv(Sq, q_block), nkb = cdiv(Skv, kv_block), wpr = cdiv(nkb, 32), kv_wpb = cdiv(Skv, 32);
  const int G = B * Hkv;
  const uint32_t* bits = block_bits;
  if (!bits) {  // BSR rows -> bitmap, validated on the device and read back once
    cudaMemPool_t pool;
    BFA_CUDA(plan_pool(&pool), "plan memory pool");
    const size_t nb = sizeof(uint32_t) * static_cast<size_t>(G) * nqb * wpr;
    BFA_CUDA(cudaMallocFromPoolAsync(reinterpret_cast<void**>(&tmp_bits), std::max<size_t>(nb, 4), pool, st),
             "block bitmap");
    BFA_CUDA(cudaMemsetAsync(tmp_bits, 0, std::max<size_t>(nb, 4), st), "clear block bitmap");
    BFA_CUDA(launch_bsr_to_bits(indptr, indices, n_indices, G, nqb, nkb, wpr, tmp_bits, P->err, st),
             "BSR bitmap kernel");
    uint32_t err = 0;
    BFA_CUDA(cudaMemcpyAsync(&err, P->err, sizeof(err), cudaMemcpyDeviceToHost, st), "read BSR status");
    BFA_CUDA(cudaStreamSynchronize(st), "BSR validation");
    if (err) {
      cleanup();
      return fail(BFA_ERR_NONCANONICAL_BSR, "BSR routing is not canonical (%s)",
                  (err & DEVERR_BSR_RANGE) ? "row offsets out of range or decreasing"
                                            : "block ids unsorted, duplicated or out of range");
    }
    bits = tmp_bits;
  }
  BFA_CUDA(launch_bits_classify(bits, kv_valid, nqb, wpr, kv_wpb, q_block, kv_block, P->causal, g_pack, P->groups,
                                P->n_groups, P->max_nqt, P->cls, st),
           "block-sparse classify kernel");
  if ((s = build_rows(P, 1))) { cleanup(); return s; }
  int32_t nnz = 0;
  BFA_CUDA(cudaMemcpyAsync(&nnz, P->row_ptr + P->n_rows, sizeof(int32_t), cudaMemcpyDeviceToHost, st), "read size");
  BFA_CUDA(cudaStreamSynchronize(st), "plan size");
  cudaMemPool_t pool;
  BFA_CUDA(plan_pool(&pool), "plan memory pool");
  BFA_CUDA(cudaMallocFromPoolAsync(&P->fine_extra,
                                   sizeof(uint32_t) * kFineWordsPerTile * static_cast<size_t>(std::max(nnz, 1)),
                                   pool, st),
           "fine-mask allocation");
  P->fine = static_cast<uint32_t*>(P->fine_extra);
  P->fine_tiles = nnz;
  BFA_CUDA(launch_bits_fine(bits, kv_valid, nqb, wpr, kv_wpb, q_block, kv_block, P->causal, g_pack, P->groups,
                            P->row_group, P->n_rows, P->row_ptr, P->kv_tile, P->part, P->fine, st),
           "block-sparse fine-mask kernel");
  if (tmp_bits) {
    cudaFreeAsync(tmp_bits, st);
    tmp_bits = nullptr;
  }
  *out = P;
  return BFA_OK;
}

}  // namespace

BFA_API bfa_status bfa_plan_predicate(const bfa_mask_term* terms, int n_terms, int B, int Sq, int Sk,
                                      const int32_t* cu_q, const int32_t* cu_k, const int32_t* seqused_k, int max_q,
                                      int max_k, bfa_plan** out, void* stream) {
  if (!out) return fail(BFA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (B <= 0) return fail(BFA_ERR_INVALID_ARG, "B=%d must be positive", B);
  if (n_terms < 0 || n_terms > BFA_MAX_MASK_TERMS)
    return fail(BFA_ERR_INVALID_ARG, "n_terms=%d must be in [0, %d]", n_terms, BFA_MAX_MASK_TERMS);
  if (n_terms > 0 && !terms) return fail(BFA_ERR_INVALID_ARG, "terms is NULL");
  if ((cu_q == nullptr) != (cu_k == nullptr))
    return fail(BFA_ERR_INVALID_ARG, "cu_seqlens_q and cu_seqlens_k must both be given or both be NULL");
  bfa_status s;
  if ((s = need_device(cu_q, "cu_seqlens_q", true)) || (s = need_device(cu_k, "cu_seqlens_k", true)) ||
      (s = need_device(seqused_k, "seqused_k", true)))
    return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bfa_plan* P = new bfa_plan();
  auto cleanup = [&]() { free_plan(P); };
  P->kind = BFA_PLAN_PREDICATE;
  P->mask_mode = MASK_PRED;
  P->varlen = cu_q != nullptr;
  P->batch = B;
  P->stream = st;
  P->n_terms = n_terms;
  if ((s = setup_seq_groups(P, B, Sq, Sk, cu_q, cu_k, seqused_k, max_q, max_k, st))) { cleanup(); return s; }
  finalize_layout(P);
  if ((s = check_capacity(P, false))) { cleanup(); return s; }
  if ((s = alloc_plan(P, false, 0, 0, 0, static_cast<int64_t>(n_terms) * 6))) { cleanup(); return s; }
  if (n_terms > 0) {
    // pageable upload of a few ints, completed before the call returns
    BFA_CUDA(cudaMemcpyAsync(P->terms, terms, sizeof(bfa_mask_term) * n_terms, cudaMemcpyHostToDevice, st),
             "upload mask terms");
  }
  BFA_CUDA(launch_pred_classify(P->terms, n_terms, P->groups, P->n_groups, P->max_nqt, P->cls, st),
           "predicate classify kernel");
  if ((s = build_rows(P))) { cleanup(); return s; }
  *out = P;
  return BFA_OK;
}

BFA_API bfa_status bfa_plan_bsr(const int32_t* indptr, const int32_t* indices, int64_t n_indices, int B, int Hkv,
                                int Sq, int Skv, int q_block, int kv_block, int causal, const uint32_t* kv_valid_bits,
                                bfa_plan** out, void* stream) {
  if (!out) return fail(BFA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (B <= 0 || Hkv <= 0 || Sq <= 0 || Skv <= 0 || n_indices < 0)
    return fail(BFA_ERR_INVALID_ARG, "bad sizes B=%d Hkv=%d Sq=%d Skv=%d n_indices=%lld", B, Hkv, Sq, Skv,
                (long long)n_indices);
  if (q_block <= 0) return fail(BFA_ERR_INVALID_ARG, "q_block=%d must be positive", q_block);
  if (!kv_block_ok(kv_block))
    return fail(BFA_ERR_INVALID_ARG, "kv_block=%d: allowed sizes are 8, 16, 32 and the multiples of 64", kv_block);
  bfa_status s;
  if ((s = need_device(indptr, "block_indptr"))) return s;
  if (n_indices > 0 && (s = need_device(indices, "block_indices"))) return s;
  if ((s = need_device(kv_valid_bits, "kv_valid_bits", true))) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (q_block != kTile || kv_block != kTile || kv_valid_bits != nullptr)
    return plan_block_sparse(indptr, indices, n_indices, nullptr, kv_valid_bits, B, Hkv, Sq, Skv, q_block, kv_block,
                             causal, out, st);
  // 128 x 128 blocks: BSR rows are tile rows; causal blocks are classified by position
  bfa_plan* P = new bfa_plan();
  auto cleanup = [&]() { free_plan(P); };
  P->kind = BFA_PLAN_BSR;
  P->mask_mode = MASK_POS;
  P->causal = causal ? 1 : 0;
  P->window = -1;
  P->batch = B;
  P->hkv = Hkv;
  P->sq = Sq;
  P->sk = Skv;
  P->stream = st;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) P->groups_h.push_back(make_group(0, Sq, 0, Skv, b, h));
  P->regular = true;
  P->regular_hkv = Hkv;
  finalize_layout(P);
  if ((s = check_capacity(P, false))) { cleanup(); return s; }
  if ((s = alloc_plan(P, false, 0, 0, 0))) { cleanup(); return s; }
  BFA_CUDA(cudaMemsetAsync(P->cls, 0, static_cast<size_t>(std::max<int64_t>(P->grid_tiles, 1)), st), "clear classes");
  BFA_CUDA(launch_bsr_classify(indptr, indices, n_indices, P->groups, P->n_groups, cdiv(Sq, kTile), P->causal, P->cls,
                               P->err, P->max_width, st),
           "BSR classify kernel");
  uint32_t err = 0;
  BFA_CUDA(cudaMemcpyAsync(&err, P->err, sizeof(err), cudaMemcpyDeviceToHost, st), "read BSR status");
  BFA_CUDA(cudaStreamSynchronize(st), "BSR validation");
  if (err) {
    cleanup();
    return fail(BFA_ERR_NONCANONICAL_BSR, "BSR routing is not canonical (%s)",
                (err & DEVERR_BSR_RANGE) ? "row offsets out of range or decreasing"
                                          : "block ids unsorted, duplicated or out of range");
  }
  if ((s = build_rows(P))) { cleanup(); return s; }
  *out = P;
  return BFA_OK;
}

BFA_API bfa_status bfa_plan_bsr_packed(const int32_t* indptr, const int32_t* indices, int64_t n_indices, int B,
                                       int Hkv, int heads_per_kv, int Sq, int Skv, int q_block, int kv_block,
                                       int causal, const uint32_t* kv_valid_bits, bfa_plan** out, void* stream) {
  if (!out) return fail(BFA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (B <= 0 || Hkv <= 0 || Sq <= 0 || Skv <= 0 || n_indices < 0)
    return fail(BFA_ERR_INVALID_ARG, "bad sizes B=%d Hkv=%d Sq=%d Skv=%d n_indices=%lld", B, Hkv, Sq, Skv,
                (long long)n_indices);
  const int G = heads_per_kv;
  if (G <= 0 || G > kTile || (G & (G - 1)) != 0)
    return fail(BFA_ERR_INVALID_ARG, "heads_per_kv=%d must be a power of two up to %d", G, kTile);
  if (q_block <= 0 || (static_cast<int64_t>(q_block) * G) % 8 != 0)
    return fail(BFA_ERR_INVALID_ARG, "q_block=%d times heads_per_kv=%d must be a positive multiple of 8", q_block, G);
  if (static_cast<int64_t>(Sq) * G >= (int64_t(1) << 31))
    return fail(BFA_ERR_CAPACITY, "Sq * heads_per_kv = %lld exceeds int32", (long long)Sq * G);
  if (!kv_block_ok(kv_block))
    return fail(BFA_ERR_INVALID_ARG, "kv_block=%d: allowed sizes are 8, 16, 32 and the multiples of 64", kv_block);
  bfa_status s;
  if ((s = need_device(indptr, "block_indptr"))) return s;
  if (n_indices > 0 && (s = need_device(indices, "block_indices"))) return s;
  if ((s = need_device(kv_valid_bits, "kv_valid_bits", true))) return s;
  return plan_block_sparse(indptr, indices, n_indices, nullptr, kv_valid_bits, B, Hkv, Sq, Skv, q_block, kv_block,
                           causal, out, static_cast<cudaStream_t>(stream), G);
}

BFA_API bfa_status bfa_plan_block_bits(const uint32_t* block_bits, int B, int Hkv, int Sq, int Skv, int q_block,
                                       int kv_block, int causal, const uint32_t* kv_valid_bits, bfa_plan** out,
                                       void* stream) {
  if (!out) return fail(BFA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (B <= 0 || Hkv <= 0 || Sq <= 0 || Skv <= 0)
    return fail(BFA_ERR_INVALID_ARG, "bad sizes B=%d Hkv=%d Sq=%d Skv=%d", B, Hkv, Sq, Skv);
  if (q_block <= 0) return fail(BFA_ERR_INVALID_ARG, "q_block=%d must be positive", q_block);
  if (!kv_block_ok(kv_block))
    return fail(BFA_ERR_INVALID_ARG, "kv_block=%d: allowed sizes are 8, 16, 32 and the multiples of 64", kv_block);
  bfa_status s;
  if ((s = need_device(block_bits, "exact_block_bits")) || (s = need_device(kv_valid_bits, "kv_valid_bits", true)))
    return s;
  return plan_block_sparse(nullptr, nullptr, 0, block_bits, kv_valid_bits, B, Hkv, Sq, Skv, q_block, kv_block, causal,
                           out, static_cast<cudaStream_t>(stream));
}

// ----------------------------------------------------------------------------
// forward launch: TMA tensor maps + kernel parameters
// ----------------------------------------------------------------------------
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  }
  return fn;
}

// 4-D map over (d, head, token, batch) of a bf16 tensor, box = 64 d x 1 head x
// 128 tokens x 1 batch, 128-byte swizzle: one 16 KB panel of a 128 x D tile.
bool make_tmap(CUtensorMap* m, const void* base, int D, int heads, int64_t tokens, int batch, int64_t s_head,
               int64_t s_tok, int64_t s_batch, std::string* why, int box_rows = kTile) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    *why = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  if (s_batch == 0 || batch == 1) s_batch = std::max<int64_t>(s_tok * std::max<int64_t>(tokens, 1), 8);
  if (s_head == 0) s_head = 8;  // a single head: any aligned stride
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(tokens),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(s_head) * 2, static_cast<cuuint64_t>(s_tok) * 2,
                           static_cast<cuuint64_t>(s_batch) * 2};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[160];
    snprintf(buf, sizeof(buf), "tensor map rejected (CUresult %d) for strides (%lld, %lld, %lld)", (int)r,
             (long long)s_head, (long long)s_tok, (long long)s_batch);
    *why = buf;
    return false;
  }
  return true;
}

// 5-D map over (d, head in group, kv head, token, batch) of a bf16 (B, S, H, D)
// tensor whose G heads of a kv head are adjacent: box = 64 d x G heads x 1 kv head
// x 128 / G tokens x 1 batch, so a box is one 128-row tile of GQA-packed rows
// (position-major, head-minor), 128-byte swizzle.
bool make_tmap_packed(CUtensorMap* m, const void* base, int D, int G, int hkv, int64_t tokens, int batch,
                      int64_t s_head, int64_t s_tok, int64_t s_batch, std::string* why) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    *why = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  if (s_batch == 0 || batch == 1) s_batch = std::max<int64_t>(s_tok * std::max<int64_t>(tokens, 1), 8);
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(G), static_cast<cuuint64_t>(hkv),
                        static_cast<cuuint64_t>(tokens), static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(s_head) * 2, static_cast<cuuint64_t>(s_head) * G * 2,
                           static_cast<cuuint64_t>(s_tok) * 2, static_cast<cuuint64_t>(s_batch) * 2};
  cuuint32_t box[5] = {64, static_cast<cuuint32_t>(G), 1, static_cast<cuuint32_t>(kTile / G), 1};
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[160];
    snprintf(buf, sizeof(buf), "packed tensor map rejected (CUresult %d) for strides (%lld, %lld, %lld)", (int)r,
             (long long)s_head, (long long)s_tok, (long long)s_batch);
    *why = buf;
    return false;
  }
  return true;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

struct PagedKV {
  const int32_t* block_table = nullptr;
  int page_size = 0, pages_per_seq = 0;
  int64_t cache_tokens = 0;  // num_pages * page_size
};

cudaError_t fwd_launch_from_host(const bfa_plan* P, const void* q, const void* k, const void* v, const int64_t* qs,
                                 const int64_t* ks, const int64_t* vs, int B, int H, int Hkv, int D, float scale,
                                 void* out, const int64_t* os, float* lse, uint64_t wait_ns, cudaStream_t st,
                                 std::string* why, const PagedKV& pg = PagedKV(), float skip_log2 = 0.f) {
  const int bq = P->varlen ? 1 : B;
  const int G = P->pack_g;
  CUtensorMap tq, tk, tv, to;
  if (G > 1) {  // GQA-packed tiles: the plan was made for G heads per kv head
    if (H != Hkv * G) {
      *why = "the plan packs " + std::to_string(G) + " query heads per kv head; H / Hkv = " +
             std::to_string(H / Hkv);
      return cudaErrorInvalidValue;
    }
    if (!make_tmap_packed(&tq, q, D, G, Hkv, P->sq, bq, qs[2], qs[1], qs[0], why) ||
        !make_tmap_packed(&to, out, D, G, Hkv, P->sq, bq, os[2], os[1], os[0], why))
      return cudaErrorInvalidValue;
  } else {
    if (!make_tmap(&tq, q, D, H, P->sq, bq, qs[2], qs[1], qs[0], why)) return cudaErrorInvalidValue;
    // the output with the query layout: whole in-range tiles leave through TMA stores
    if (!make_tmap(&to, out, D, H, P->sq, bq, os[2], os[1], P->varlen ? 0 : os[0], why)) return cudaErrorInvalidValue;
  }
  if (pg.page_size == 0) {
    if (!make_tmap(&tk, k, D, Hkv, P->sk, bq, ks[2], ks[1], ks[0], why) ||
        !make_tmap(&tv, v, D, Hkv, P->sk, bq, vs[2], vs[1], vs[0], why))
      return cudaErrorInvalidValue;
  } else {  // the cache as one token axis; boxes of one page (at most one tile)
    const int rows = std::min(pg.page_size, static_cast<int>(kTile));
    if (!make_tmap(&tk, k, D, Hkv, pg.cache_tokens, 1, ks[2], ks[1], 0, why, rows) ||
        !make_tmap(&tv, v, D, Hkv, pg.cache_tokens, 1, vs[2], vs[1], 0, why, rows))
      return cudaErrorInvalidValue;
  }
  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.plan.groups = P->groups;
  p.plan.row_group = P->row_group;
  p.plan.row_ptr = P->row_ptr;
  p.plan.kv_tile = P->kv_tile;
  p.plan.part = P->part;
  p.plan.fine = P->fine;
  p.plan.order = P->order;
  p.plan.row_work = P->row_work;
  p.plan.pair_work = P->pair_work;
  p.plan.qid = P->qid;
  p.plan.qvalid = P->qvalid;
  p.plan.kid = P->kid;
  p.plan.kbits = P->kbits;
  p.plan.terms = P->terms;
  p.plan.n_terms = P->n_terms;
  p.plan.err = P->err;
  p.plan.cap_tiles = std::max<int64_t>(P->grid_tiles, 1);
  p.plan.cap_fine = std::max<int64_t>(P->fine_tiles, 1);
  p.plan.cap_qid = P->cap_qid;
  p.plan.cap_kid = P->cap_kid;
  p.plan.cap_kbits = P->cap_kbits;
  p.plan.n_rows = P->n_rows;
  p.plan.n_groups = P->n_groups;
  p.plan.mask_mode = P->mask_mode;
  p.plan.causal = P->causal;
  p.plan.window = P->window;
  p.plan.kind = P->kind;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.D = D;
  // packed plans hold every head of a kv head in their rows: one replica per row
  p.rep = P->kind == BFA_PLAN_DENSE ? B * H : (P->kind == BFA_PLAN_BSR ? (G > 1 ? 1 : H / Hkv) : H);
  p.pack_g = G;
  p.pack_shift = 0;
  while ((1 << p.pack_shift) < G) ++p.pack_shift;
  p.plan.pair_row = P->pair_row;
  p.plan.pair_order = P->pair_order;
  p.plan.n_pairs = P->n_pairs;
  // A CTA runs two query tiles that share K/V: two heads of one kv head on the
  // same row when the GQA group is even (identical key lists), else two
  // consecutive query tiles of one head.
  p.pair_heads = (G == 1 && (H / Hkv) % 2 == 0) ? 1 : 0;
  const int64_t units = p.pair_heads ? P->n_rows : P->n_pairs;
  const int64_t items = p.pair_heads ? p.rep / 2 : p.rep;
  // Keep enough replica units of a row together to fill about two waves of
  // CTAs, but no more kv heads than stay resident in L2 (about 64 MB).
  const int64_t waves = 2LL * sm_count();
  int64_t chunk = std::min<int64_t>(items, std::max<int64_t>(1, (waves + units - 1) / std::max<int64_t>(units, 1)));
  const int64_t kv_head_bytes = std::max<int64_t>(1, static_cast<int64_t>(P->sk) * D * 4);
  const int64_t l2_kv_heads = std::max<int64_t>(1, (64LL << 20) / kv_head_bytes);
  const int64_t units_per_kv_head = G > 1 ? 1 : (p.pair_heads ? std::max(1, (H / Hkv) / 2) : std::max(1, H / Hkv));
  chunk = std::max<int64_t>(1, std::min<int64_t>(chunk, l2_kv_heads * units_per_kv_head));
  p.head_chunk = static_cast<int>(chunk);
  p.varlen = P->varlen;
  p.Sq_lse = P->sq;
  const float sc = (scale > 0.f) ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale_log2 = sc * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.o_sb = P->varlen ? 0 : os[0];
  p.o_ss = os[1];
  p.o_sh = os[2];
  p.lse = lse;
  p.wait_ns = wait_ns;
  p.block_table = pg.block_table;
  p.page_size = pg.page_size;
  p.pages_per_seq = pg.pages_per_seq;
  p.skip_log2 = skip_log2;
  const int64_t n_work = units * items;
  return launch_fwd(D, tq, tk, tv, to, p, n_work, st);
}

}  // namespace

namespace {

bfa_status fwd_checked(const bfa_plan* P, const void* q, const void* k, const void* v, const int64_t qs[3],
                       const int64_t ks[3], const int64_t vs[3], int B, int H, int Hkv, int D, float scale, void* out,
                       const int64_t os[3], float* lse, void* stream, float skip_log2) {
  if (!P) return fail(BFA_ERR_INVALID_ARG, "plan is NULL");
  if (!qs || !ks || !vs || !os) return fail(BFA_ERR_INVALID_ARG, "strides are NULL");
  if (D != 64 && D != 128) return fail(BFA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", D);
  if (H <= 0 || Hkv <= 0 || H % Hkv != 0) return fail(BFA_ERR_INVALID_ARG, "H=%d must be a positive multiple of Hkv=%d", H, Hkv);
  if (B <= 0) return fail(BFA_ERR_INVALID_ARG, "B=%d must be positive", B);
  if (P->kind != BFA_PLAN_DENSE && B != P->batch)
    return fail(BFA_ERR_INVALID_ARG, "B=%d does not match the plan's %d", B, P->batch);
  if (P->kind == BFA_PLAN_BSR && Hkv != P->hkv)
    return fail(BFA_ERR_INVALID_ARG, "Hkv=%d does not match the BSR routing's %d", Hkv, P->hkv);
  bfa_status s;
  if ((s = need_device(q, "q")) || (s = need_device(k, "k")) || (s = need_device(v, "v")) ||
      (s = need_device(out, "out")) || (s = need_device(lse, "lse", true)))
    return s;
  const int64_t* all[4] = {qs, ks, vs, os};
  for (int t = 0; t < 4; ++t)
    for (int i = 0; i < 3; ++i) {
      if (P->varlen && i == 0) continue;
      if (all[t][i] < 0 || all[t][i] % 8 != 0)
        return fail(BFA_ERR_INVALID_ARG, "stride %lld is not a non-negative multiple of 8 elements", (long long)all[t][i]);
    }
  const void* ptrs[4] = {q, k, v, out};
  for (int t = 0; t < 4; ++t)
    if (reinterpret_cast<uintptr_t>(ptrs[t]) & 15u) return fail(BFA_ERR_INVALID_ARG, "tensor base is not 16-byte aligned");
  std::string why;
  cudaError_t e = fwd_launch_from_host(P, q, k, v, qs, ks, vs, B, H, Hkv, D, scale, out, os, lse, g_wait_ns,
                                       static_cast<cudaStream_t>(stream), &why, PagedKV(), skip_log2);
  if (e != cudaSuccess) {
    if (!why.empty()) return fail(BFA_ERR_INVALID_ARG, "%s", why.c_str());
    return cuda_fail(e, "forward kernel");
  }
  return BFA_OK;
}

}  // namespace

namespace {

// Backward: preprocess (D, LSE * log2 e) -> dQ pass over the plan's rows -> dK/dV
// pass over its key-tile columns.  The workspace comes from the plan pool in
// stream order and is returned after the kernels.
bfa_status bwd_launch_from_host(bfa_plan* P, const void* q, const void* k, const void* v, const void* out,
                                const void* dout, const float* lse, const int64_t* qs, const int64_t* ks,
                                const int64_t* vs, const int64_t* os, const int64_t* dos, int B, int H, int Hkv,
                                int D, float scale, void* dq, void* dk, void* dv, const int64_t* dqs,
                                const int64_t* dks, const int64_t* dvs, cudaStream_t st) {
  std::string why;
  const int bq = P->varlen ? 1 : B;
  const int G = P->pack_g;
  CUtensorMap tq, tdo, tk, tv;
  const bool qmaps = G > 1 ? (make_tmap_packed(&tq, q, D, G, Hkv, P->sq, bq, qs[2], qs[1], qs[0], &why) &&
                              make_tmap_packed(&tdo, dout, D, G, Hkv, P->sq, bq, dos[2], dos[1], dos[0], &why))
                           : (make_tmap(&tq, q, D, H, P->sq, bq, qs[2], qs[1], qs[0], &why) &&
                              make_tmap(&tdo, dout, D, H, P->sq, bq, dos[2], dos[1], dos[0], &why));
  if (!qmaps ||
      !make_tmap(&tk, k, D, Hkv, P->sk, bq, ks[2], ks[1], ks[0], &why) ||
      !make_tmap(&tv, v, D, Hkv, P->sk, bq, vs[2], vs[1], vs[0], &why))
    return fail(BFA_ERR_INVALID_ARG, "%s", why.c_str());
  bfa_status s = ensure_cols(P, st);
  if (s != BFA_OK) return s;
  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.plan.groups = P->groups;
  p.plan.row_group = P->row_group;
  p.plan.row_ptr = P->row_ptr;
  p.plan.kv_tile = P->kv_tile;
  p.plan.part = P->part;
  p.plan.fine = P->fine;
  p.plan.order = P->order;
  p.plan.row_work = P->row_work;
  p.plan.pair_work = P->pair_work;
  p.plan.qid = P->qid;
  p.plan.qvalid = P->qvalid;
  p.plan.kid = P->kid;
  p.plan.kbits = P->kbits;
  p.plan.terms = P->terms;
  p.plan.n_terms = P->n_terms;
  p.plan.err = P->err;
  p.plan.cap_tiles = std::max<int64_t>(P->grid_tiles, 1);
  p.plan.cap_fine = std::max<int64_t>(P->fine_tiles, 1);
  p.plan.cap_qid = P->cap_qid;
  p.plan.cap_kid = P->cap_kid;
  p.plan.cap_kbits = P->cap_kbits;
  p.plan.n_rows = P->n_rows;
  p.plan.n_groups = P->n_groups;
  p.plan.mask_mode = P->mask_mode;
  p.plan.causal = P->causal;
  p.plan.window = P->window;
  p.plan.kind = P->kind;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.D = D;
  // packed plans hold every head of a kv head in their rows: one replica per row
  p.rep = P->kind == BFA_PLAN_DENSE ? B * H : (P->kind == BFA_PLAN_BSR ? (G > 1 ? 1 : H / Hkv) : H);
  p.rep_kv = P->kind == BFA_PLAN_DENSE ? B * Hkv : (P->kind == BFA_PLAN_BSR ? 1 : Hkv);
  p.pack_g = G;
  p.pack_shift = 0;
  while ((1 << p.pack_shift) < G) ++p.pack_shift;
  const int n_cols = plan_n_cols(P);
  const int64_t waves = 2LL * sm_count();
  auto chunk_for = [&](int64_t units, int64_t items) {
    return std::min<int64_t>(items, std::max<int64_t>(1, (waves + units - 1) / std::max<int64_t>(units, 1)));
  };
  p.head_chunk = static_cast<int>(chunk_for(P->n_rows, p.rep));
  // The fused pass keeps one kv replica's columns together on batched and dense
  // plans, so that the fp32 dQ rows its columns sum into stay in L2 (measured: 3-6 %
  // on the union mask, about 1 % on block-causal GQA, even on causal and BSR); on
  // varlen plans the two passes' order, which spreads the columns over two kv
  // heads, measured faster.
  const bool fused_order = D == 128 && !g_bwd_deterministic && !P->varlen;
  p.kv_chunk = fused_order ? 1 : static_cast<int>(chunk_for(n_cols, p.rep_kv));
  p.varlen = P->varlen;
  p.Sq_lse = P->sq;
  const float sc = (scale > 0.f) ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale = sc;
  p.scale_log2 = sc * 1.4426950408889634f;
  p.out = static_cast<const __nv_bfloat16*>(out);
  p.o_sb = P->varlen ? 0 : os[0];
  p.o_ss = os[1];
  p.o_sh = os[2];
  p.dout = static_cast<const __nv_bfloat16*>(dout);
  p.do_sb = P->varlen ? 0 : dos[0];
  p.do_ss = dos[1];
  p.do_sh = dos[2];
  p.lse = lse;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dq_sb = P->varlen ? 0 : dqs[0];
  p.dq_ss = dqs[1];
  p.dq_sh = dqs[2];
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dk_sb = P->varlen ? 0 : dks[0];
  p.dk_ss = dks[1];
  p.dk_sh = dks[2];
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.dv_sb = P->varlen ? 0 : dvs[0];
  p.dv_ss = dvs[1];
  p.dv_sh = dvs[2];
  p.col0 = P->col0;
  p.col_group = P->col_group;
  p.col_ptr = P->col_ptr;
  p.q_tile = P->q_tile;
  p.tpart = P->tpart;
  p.col_order = P->col_order;
  p.n_cols = n_cols;
  p.wait_ns = g_wait_ns;
  const int64_t ws_rows = static_cast<int64_t>(p.rep) * P->n_rows * kTile;
  // D = 128 runs the fused pass, which also needs the fp32 dQ sums (D floats a row),
  // unless reproducible sums were asked for
  const bool fused = D == 128 && !g_bwd_deterministic;
  const int64_t ws_floats = ws_rows * (2 + (fused ? D : 0));
  void* ws = nullptr;
  auto cleanup = [&]() {
    if (ws) cudaFreeAsync(ws, st);
  };
  if (ws_rows > 0) {
    cudaMemPool_t pool;
    BFA_CUDA(plan_pool(&pool), "plan memory pool");
    cudaError_t e = cudaMallocFromPoolAsync(&ws, static_cast<size_t>(ws_floats) * sizeof(float), pool, st);
    if (e != cudaSuccess) {
      ws = nullptr;
      return fail(BFA_ERR_CAPACITY, "backward workspace of %lld bytes: %s", (long long)(ws_floats * 4),
                  cudaGetErrorString(e));
    }
    p.ws_lse2 = static_cast<float*>(ws);
    p.ws_d = p.ws_lse2 + ws_rows;
    p.dq_acc = fused ? p.ws_d + ws_rows : nullptr;
  }
  BFA_CUDA(launch_bwd_prep(p, st), "backward preprocess kernel");
  if (fused) {
    BFA_CUDA(launch_bwd_fused(tk, tv, tq, tdo, p, static_cast<int64_t>(n_cols) * p.rep_kv, st), "fused backward kernel");
    BFA_CUDA(launch_bwd_dq_store(p, st), "dQ store kernel");
  } else {
    BFA_CUDA(launch_bwd_dq(D, tq, tdo, tk, tv, p, static_cast<int64_t>(P->n_rows) * p.rep, st), "dQ kernel");
    BFA_CUDA(launch_bwd_dkdv(D, tk, tv, tq, tdo, p, static_cast<int64_t>(n_cols) * p.rep_kv, st), "dK/dV kernel");
  }
  cleanup();
  return BFA_OK;
}

}  // namespace

BFA_API bfa_status bfa_bwd(const bfa_plan* Pc, const void* q, const void* k, const void* v, const void* out,
                           const void* dout, const float* lse, const int64_t qs[3], const int64_t ks[3],
                           const int64_t vs[3], const int64_t os[3], const int64_t dos[3], int B, int H, int Hkv,
                           int D, float scale, void* dq, void* dk, void* dv, const int64_t dqs[3],
                           const int64_t dks[3], const int64_t dvs[3], void* stream) {
  if (!Pc) return fail(BFA_ERR_INVALID_ARG, "plan is NULL");
  bfa_plan* P = const_cast<bfa_plan*>(Pc);  // the transposed lists are a cache of the plan
  if (!qs || !ks || !vs || !os || !dos || !dqs || !dks || !dvs) return fail(BFA_ERR_INVALID_ARG, "strides are NULL");
  if (D != 64 && D != 128) return fail(BFA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", D);
  if (H <= 0 || Hkv <= 0 || H % Hkv != 0) return fail(BFA_ERR_INVALID_ARG, "H=%d must be a positive multiple of Hkv=%d", H, Hkv);
  if (B <= 0) return fail(BFA_ERR_INVALID_ARG, "B=%d must be positive", B);
  if (P->kind != BFA_PLAN_DENSE && B != P->batch)
    return fail(BFA_ERR_INVALID_ARG, "B=%d does not match the plan's %d", B, P->batch);
  if (P->kind == BFA_PLAN_BSR && Hkv != P->hkv)
    return fail(BFA_ERR_INVALID_ARG, "Hkv=%d does not match the BSR routing's %d", Hkv, P->hkv);
  if (P->pack_g > 1 && H != Hkv * P->pack_g)
    return fail(BFA_ERR_INVALID_ARG, "the plan packs %d query heads per kv head; H / Hkv = %d", P->pack_g, H / Hkv);
  if (!lse) return fail(BFA_ERR_INVALID_ARG, "lse is required by the backward");
  bfa_status s;
  if ((s = need_device(q, "q")) || (s = need_device(k, "k")) || (s = need_device(v, "v")) ||
      (s = need_device(out, "out")) || (s = need_device(dout, "dout")) || (s = need_device(lse, "lse")) ||
      (s = need_device(dq, "dq")) || (s = need_device(dk, "dk")) || (s = need_device(dv, "dv")))
    return s;
  const int64_t* all[8] = {qs, ks, vs, os, dos, dqs, dks, dvs};
  for (int t = 0; t < 8; ++t)
    for (int i = 0; i < 3; ++i) {
      if (P->varlen && i == 0) continue;
      if (all[t][i] < 0 || all[t][i] % 8 != 0)
        return fail(BFA_ERR_INVALID_ARG, "stride %lld is not a non-negative multiple of 8 elements", (long long)all[t][i]);
    }
  const void* ptrs[8] = {q, k, v, out, dout, dq, dk, dv};
  for (int t = 0; t < 8; ++t)
    if (reinterpret_cast<uintptr_t>(ptrs[t]) & 15u) return fail(BFA_ERR_INVALID_ARG, "tensor base is not 16-byte aligned");
  return bwd_launch_from_host(P, q, k, v, out, dout, lse, qs, ks, vs, os, dos, B, H, Hkv, D, scale, dq, dk, dv, dqs,
                              dks, dvs, static_cast<cudaStream_t>(stream));
}

BFA_API bfa_status bfa_fwd(const bfa_plan* P, const void* q, const void* k, const void* v, const int64_t qs[3],
                           const int64_t ks[3], const int64_t vs[3], int B, int H, int Hkv, int D, float scale,
                           void* out, const int64_t os[3], float* lse, void* stream) {
  return fwd_checked(P, q, k, v, qs, ks, vs, B, H, Hkv, D, scale, out, os, lse, stream, 0.f);
}

BFA_API bfa_status bfa_fwd_approx(const bfa_plan* P, const void* q, const void* k, const void* v,
                                  const int64_t qs[3], const int64_t ks[3], const int64_t vs[3], int B, int H,
                                  int Hkv, int D, float scale, float softmax_threshold, void* out,
                                  const int64_t os[3], float* lse, void* stream) {
  if (!(softmax_threshold > 0.f))
    return fail(BFA_ERR_INVALID_ARG, "softmax_threshold must be positive (use bfa_fwd for the exact result)");
  return fwd_checked(P, q, k, v, qs, ks, vs, B, H, Hkv, D, scale, out, os, lse, stream,
                     softmax_threshold * 1.4426950408889634f);
}

BFA_API bfa_status bfa_fwd_paged(const bfa_plan* P, const void* q, const int64_t q_strides[3], const void* k_cache,
                                 const void* v_cache, const int64_t cache_strides[3], int64_t num_pages, int page_size,
                                 const int32_t* block_table, int pages_per_seq, int B, int H, int Hkv, int D,
                                 float scale, void* out, const int64_t o_strides[3], float* lse, void* stream) {
  if (!P) return fail(BFA_ERR_INVALID_ARG, "plan is NULL");
  if (!q_strides || !cache_strides || !o_strides) return fail(BFA_ERR_INVALID_ARG, "strides are NULL");
  if (D != 64 && D != 128) return fail(BFA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", D);
  if (H <= 0 || Hkv <= 0 || H % Hkv != 0) return fail(BFA_ERR_INVALID_ARG, "H=%d must be a positive multiple of Hkv=%d", H, Hkv);
  if (B <= 0) return fail(BFA_ERR_INVALID_ARG, "B=%d must be positive", B);
  if (P->kind != BFA_PLAN_DENSE && B != P->batch)
    return fail(BFA_ERR_INVALID_ARG, "B=%d does not match the plan's %d", B, P->batch);
  if (P->kind == BFA_PLAN_BSR && Hkv != P->hkv)
    return fail(BFA_ERR_INVALID_ARG, "Hkv=%d does not match the BSR routing's %d", Hkv, P->hkv);
  if (!(page_size == 8 || page_size == 16 || page_size == 32 || page_size == 64 ||
        (page_size > 0 && page_size % kTile == 0)))
    return fail(BFA_ERR_INVALID_ARG, "page_size=%d must be 8, 16, 32, 64 or a multiple of 128", page_size);
  if (num_pages <= 0 || pages_per_seq <= 0) return fail(BFA_ERR_INVALID_ARG, "num_pages / pages_per_seq must be positive");
  int max_k = 0;
  for (const auto& g : P->groups_h) max_k = std::max(max_k, g.k_len);
  if (static_cast<int64_t>(pages_per_seq) * page_size < max_k)
    return fail(BFA_ERR_INVALID_ARG, "pages_per_seq * page_size = %lld is below the plan's %d keys",
                (long long)pages_per_seq * page_size, max_k);
  if (cache_strides[0] != static_cast<int64_t>(page_size) * cache_strides[1])
    return fail(BFA_ERR_INVALID_ARG, "cache pages must be contiguous (page stride = page_size * token stride)");
  if (num_pages * page_size >= (int64_t(1) << 31)) return fail(BFA_ERR_CAPACITY, "cache too large");
  bfa_status s;
  if ((s = need_device(q, "q")) || (s = need_device(k_cache, "k_cache")) || (s = need_device(v_cache, "v_cache")) ||
      (s = need_device(block_table, "block_table")) || (s = need_device(out, "out")) ||
      (s = need_device(lse, "lse", true)))
    return s;
  const int64_t* all[3] = {q_strides, cache_strides, o_strides};
  for (int t = 0; t < 3; ++t)
    for (int i = 0; i < 3; ++i) {
      if ((P->varlen || t == 1) && i == 0) continue;
      if (all[t][i] < 0 || all[t][i] % 8 != 0)
        return fail(BFA_ERR_INVALID_ARG, "stride %lld is not a non-negative multiple of 8 elements", (long long)all[t][i]);
    }
  const void* ptrs[4] = {q, k_cache, v_cache, out};
  for (int t = 0; t < 4; ++t)
    if (reinterpret_cast<uintptr_t>(ptrs[t]) & 15u) return fail(BFA_ERR_INVALID_ARG, "tensor base is not 16-byte aligned");
  PagedKV pg;
  pg.block_table = block_table;
  pg.page_size = page_size;
  pg.pages_per_seq = pages_per_seq;
  pg.cache_tokens = num_pages * page_size;
  std::string why;
  cudaError_t e = fwd_launch_from_host(P, q, k_cache, v_cache, q_strides, cache_strides, cache_strides, B, H, Hkv, D,
                                       scale, out, o_strides, lse, g_wait_ns, static_cast<cudaStream_t>(stream), &why,
                                       pg);
  if (e != cudaSuccess) {
    if (!why.empty()) return fail(BFA_ERR_INVALID_ARG, "%s", why.c_str());
    return cuda_fail(e, "forward kernel");
  }
  return BFA_OK;
}

BFA_API bfa_status bfa_plan_get_info(const bfa_plan* P, bfa_plan_info* info) {
  if (!P || !info) return fail(BFA_ERR_INVALID_ARG, "NULL argument");
  info->kind = P->kind;
  info->varlen = P->varlen;
  info->n_groups = P->n_groups;
  info->n_rows = P->n_rows;
  info->grid_tiles = P->grid_tiles;
  info->batch = P->kind == BFA_PLAN_DENSE ? 0 : P->batch;
  info->hkv = P->hkv;
  info->sq = P->sq;
  info->sk = P->sk;
  info->max_kv_tiles = P->max_nkt;
  info->window_left = P->window;
  info->causal = P->causal;
  info->n_pairs = P->n_pairs;
  info->packed_fine = P->mask_mode == MASK_BITS ? 1 : 0;
  info->n_cols = plan_n_cols(P);
  info->heads_per_kv = P->pack_g;
  return BFA_OK;
}

BFA_API bfa_status bfa_plan_stats(const bfa_plan* P, int64_t* n_full, int64_t* n_partial, int64_t* n_empty,
                                  void* stream) {
  if (!P) return fail(BFA_ERR_INVALID_ARG, "plan is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::vector<uint8_t> cls(static_cast<size_t>(P->grid_tiles));
  auto cleanup = []() {};
  if (P->grid_tiles > 0) {
    BFA_CUDA(cudaMemcpyAsync(cls.data(), P->cls, cls.size(), cudaMemcpyDeviceToHost, st), "read classes");
  }
  BFA_CUDA(cudaStreamSynchronize(st), "plan stats");
  int64_t c[3] = {0, 0, 0};
  for (uint8_t x : cls) c[x < 3 ? x : 0]++;
  if (n_empty) *n_empty = c[0];
  if (n_partial) *n_partial = c[1];
  if (n_full) *n_full = c[2];
  return BFA_OK;
}

BFA_API bfa_status bfa_plan_export(const bfa_plan* P, int32_t* row_ptr, int32_t* kv_tile, uint8_t* partial,
                                   uint32_t* fine, int32_t* order, uint8_t* classes, void* stream) {
  if (!P) return fail(BFA_ERR_INVALID_ARG, "plan is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto cleanup = []() {};
  std::vector<int32_t> rp(P->n_rows + 1);
  BFA_CUDA(cudaMemcpyAsync(rp.data(), P->row_ptr, sizeof(int32_t) * rp.size(), cudaMemcpyDeviceToHost, st), "read row_ptr");
  BFA_CUDA(cudaStreamSynchronize(st), "export");
  const int64_t nnz = rp[P->n_rows];
  std::vector<int32_t> part(nnz);
  if (nnz > 0) BFA_CUDA(cudaMemcpyAsync(part.data(), P->part, sizeof(int32_t) * nnz, cudaMemcpyDeviceToHost, st), "read parts");
  if (row_ptr) std::memcpy(row_ptr, rp.data(), sizeof(int32_t) * rp.size());
  if (kv_tile && nnz > 0)
    BFA_CUDA(cudaMemcpyAsync(kv_tile, P->kv_tile, sizeof(int32_t) * nnz, cudaMemcpyDeviceToHost, st), "read lists");
  if (order && P->n_rows > 0)
    BFA_CUDA(cudaMemcpyAsync(order, P->order, sizeof(int32_t) * P->n_rows, cudaMemcpyDeviceToHost, st), "read order");
  if (classes && P->grid_tiles > 0)
    BFA_CUDA(cudaMemcpyAsync(classes, P->cls, static_cast<size_t>(P->grid_tiles), cudaMemcpyDeviceToHost, st), "read classes");
  std::vector<uint32_t> fine_all;
  const bool want_fine = fine && P->mask_mode == MASK_BITS && P->fine_tiles > 0;
  if (want_fine) {
    fine_all.resize(static_cast<size_t>(P->fine_tiles) * kFineWordsPerTile);
    BFA_CUDA(cudaMemcpyAsync(fine_all.data(), P->fine, fine_all.size() * sizeof(uint32_t), cudaMemcpyDeviceToHost, st),
             "read fine masks");
  }
  BFA_CUDA(cudaStreamSynchronize(st), "export");
  int64_t np = 0;
  for (int64_t e = 0; e < nnz; ++e) {
    if (partial) partial[e] = part[e] >= 0 ? 1 : 0;
    if (part[e] >= 0) {
      if (want_fine)
        std::memcpy(fine + np * kFineWordsPerTile, fine_all.data() + static_cast<int64_t>(part[e]) * kFineWordsPerTile,
                    sizeof(uint32_t) * kFineWordsPerTile);
      ++np;
    }
  }
  return BFA_OK;
}

BFA_API bfa_status bfa_plan_export_pairs(const bfa_plan* P, int32_t* pair_row, int32_t* pair_order, void* stream) {
  if (!P) return fail(BFA_ERR_INVALID_ARG, "plan is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto cleanup = []() {};
  if (P->n_pairs > 0) {
    if (pair_row)
      BFA_CUDA(cudaMemcpyAsync(pair_row, P->pair_row, sizeof(int32_t) * P->n_pairs, cudaMemcpyDeviceToHost, st),
               "read pairs");
    if (pair_order)
      BFA_CUDA(cudaMemcpyAsync(pair_order, P->pair_order, sizeof(int32_t) * P->n_pairs, cudaMemcpyDeviceToHost, st),
               "read pair order");
  }
  BFA_CUDA(cudaStreamSynchronize(st), "export pairs");
  return BFA_OK;
}

BFA_API bfa_status bfa_plan_export_cols(const bfa_plan* Pc, int32_t* col_ptr, int32_t* q_tile, int32_t* tpart,
                                        int32_t* col_order, void* stream) {
  if (!Pc) return fail(BFA_ERR_INVALID_ARG, "plan is NULL");
  bfa_plan* P = const_cast<bfa_plan*>(Pc);  // the transposed lists are a cache of the plan
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto cleanup = []() {};
  bfa_status s = ensure_cols(P, st);
  if (s != BFA_OK) return s;
  const int n_cols = plan_n_cols(P);
  int32_t n_listed = 0;
  BFA_CUDA(cudaMemcpyAsync(&n_listed, P->col_ptr + n_cols, sizeof(int32_t), cudaMemcpyDeviceToHost, st),
           "read column count");
  BFA_CUDA(cudaStreamSynchronize(st), "export columns");
  if (col_ptr)
    BFA_CUDA(cudaMemcpyAsync(col_ptr, P->col_ptr, sizeof(int32_t) * (n_cols + 1), cudaMemcpyDeviceToHost, st),
             "read col_ptr");
  if (n_listed > 0 && q_tile)
    BFA_CUDA(cudaMemcpyAsync(q_tile, P->q_tile, sizeof(int32_t) * n_listed, cudaMemcpyDeviceToHost, st), "read q_tile");
  if (n_listed > 0 && tpart)
    BFA_CUDA(cudaMemcpyAsync(tpart, P->tpart, sizeof(int32_t) * n_listed, cudaMemcpyDeviceToHost, st), "read tpart");
  if (n_cols > 0 && col_order)
    BFA_CUDA(cudaMemcpyAsync(col_order, P->col_order, sizeof(int32_t) * n_cols, cudaMemcpyDeviceToHost, st),
             "read col_order");
  BFA_CUDA(cudaStreamSynchronize(st), "export columns");
  return BFA_OK;
}

BFA_API bfa_status bfa_plan_device_status(const bfa_plan* P, void* stream) {
  if (!P) return fail(BFA_ERR_INVALID_ARG, "plan is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto cleanup = []() {};
  uint32_t err = 0;
  if (kChecked) {  // the guard bytes after every plan array must be intact
    BFA_CUDA(launch_check_guards(P->slab, P->guard_offs, P->n_guards, kGuardBytes, kGuardByte, P->err, st),
             "guard check kernel");
    if (P->cols_slab)
      BFA_CUDA(launch_check_guards(P->cols_slab, P->col_guard_offs, P->n_col_guards, kGuardBytes, kGuardByte, P->err,
                                   st),
               "guard check kernel");
  }
  BFA_CUDA(cudaMemcpyAsync(&err, P->err, sizeof(err), cudaMemcpyDeviceToHost, st), "read device status");
  BFA_CUDA(cudaStreamSynchronize(st), "device status");
  if (err & (DEVERR_BOUNDS | DEVERR_GUARD)) {
    BFA_CUDA(cudaMemsetAsync(P->err, 0, sizeof(uint32_t), st), "clear device status");
    BFA_CUDA(cudaStreamSynchronize(st), "device status");
    return fail(BFA_ERR_BOUNDS, "checked build: %s%s", (err & DEVERR_BOUNDS) ? "an index left its array " : "",
                (err & DEVERR_GUARD) ? "guard bytes after a plan array were overwritten" : "");
  }
  if (err & DEVERR_TIMEOUT) {
    BFA_CUDA(cudaMemsetAsync(P->err, 0, sizeof(uint32_t), st), "clear device status");
    BFA_CUDA(cudaStreamSynchronize(st), "device status");
    return fail(BFA_ERR_TIMEOUT, "a device-side wait exceeded its bound");
  }
  return BFA_OK;
}

BFA_API void bfa_plan_destroy(bfa_plan* P) { free_plan(P); }

BFA_API bfa_status bfa_selftest_wait_timeout(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* d = nullptr;
  auto cleanup = [&]() {
    if (d) cudaFreeAsync(d, st);
  };
  BFA_CUDA(cudaMallocAsync(&d, sizeof(uint32_t), st), "selftest alloc");
  BFA_CUDA(cudaMemsetAsync(d, 0, sizeof(uint32_t), st), "selftest clear");
  BFA_CUDA(launch_wait_selftest(d, g_wait_ns, st), "selftest kernel");
  uint32_t h = 0;
  BFA_CUDA(cudaMemcpyAsync(&h, d, sizeof(h), cudaMemcpyDeviceToHost, st), "selftest read");
  BFA_CUDA(cudaStreamSynchronize(st), "selftest");
  cleanup();
  if (h & DEVERR_TIMEOUT) return fail(BFA_ERR_TIMEOUT, "bounded wait gave up as designed");
  return BFA_OK;
}

// ----------------------------------------------------------------------------
// Dense planner that allocates nothing
// ----------------------------------------------------------------------------
// For callers that cannot let the library allocate device memory, for example a
// serving process whose memory manager has reserved the whole GPU up front, or
// code that must keep a fixed, known device-memory footprint.  The caller passes
// the mask and every output buffer; the planner's own scratch (the group table,
// the row -> group map and the per-row tile counts) lives in the file-scope
// device array below, which every GPU that loads the library holds until the
// process exits.
namespace {

constexpr int kNoAllocMaxRows = BFA_NOALLOC_MAX_ROWS;
constexpr size_t kNoAllocScratchBytes = 256 + 2 * sizeof(int32_t) * kNoAllocMaxRows;
static_assert(sizeof(GroupInfo) <= 256, "group table slot");

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device (set up once per
// device, with that device current).  In host code the array's name is only a
// host-side stand-in, so the address must come from cudaGetSymbolAddress.
bfa_status noalloc_scratch(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "current device");
  if (dev < 0 || dev >= 64) return fail(BFA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "scratch symbol address");
    g_noalloc_ptr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return BFA_OK;
}

}  // namespace

BFA_API bfa_status bfa_plan_dense_noalloc(const uint8_t* mask, int64_t ld, int Sq, int Sk, uint8_t* classes,
                                          int32_t* row_ptr, int32_t* kv_tile, int32_t* part, uint32_t* fine,
                                          int32_t* order, void* stream) {
  if (Sq <= 0 || Sk <= 0) return fail(BFA_ERR_INVALID_ARG, "Sq=%d Sk=%d must be positive", Sq, Sk);
  if (ld < Sk) return fail(BFA_ERR_INVALID_ARG, "mask_row_stride %lld < Sk %d", (long long)ld, Sk);
  const int nqt = cdiv(Sq, kTile), nkt = cdiv(Sk, kTile);
  if (nqt > kNoAllocMaxRows || nkt > BFA_NOALLOC_MAX_KV_TILES)
    return fail(BFA_ERR_CAPACITY, "%d x %d tiles exceed the no-allocation limits (%d query tiles, %d key tiles)",
                nqt, nkt, kNoAllocMaxRows, BFA_NOALLOC_MAX_KV_TILES);
  bfa_status s;
  if ((s = need_device(mask, "mask")) || (s = need_device(classes, "classes")) ||
      (s = need_device(row_ptr, "row_ptr")) || (s = need_device(kv_tile, "kv_tile")) ||
      (s = need_device(part, "part")) || (s = need_device(fine, "fine")) || (s = need_device(order, "order")))
    return s;
  uint8_t* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch))) return s;
  GroupInfo* groups = reinterpret_cast<GroupInfo*>(scratch);
  int32_t* row_group = reinterpret_cast<int32_t*>(scratch + 256);
  int32_t* row_cnt = row_group + kNoAllocMaxRows;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto cleanup = []() {};
  // every scratch word the kernels read is written first in this call, so the
  // previous call's contents never leak into this one
  GroupInfo g = make_group(0, Sq, 0, Sk, -1, -1);
  g.row0 = 0;
  g.cls_off = 0;
  BFA_CUDA(launch_init_regular_groups(g, 1, 1, 0, 0, groups, row_group, nqt, st), "group table kernel");
  BFA_CUDA(launch_dense_classify(mask, ld, Sq, Sk, classes, fine, st), "dense classify kernel");
  BFA_CUDA(launch_rows(groups, row_group, classes, nqt, nkt, row_cnt, row_ptr, kv_tile, part, order, st),
           "plan rows kernel");
  return BFA_OK;
}
