// C ABI of libbbattn.so: validation, the random block table, workspace
// sizing and kernel dispatch.  See include/bb_attn.h for the contract.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "common.cuh"

namespace bb {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

WsLayout ws_layout(const Problem& p, int pass) {
  WsLayout w{};
  size_t off = 0;
  w.status_off = off;
  off += 256;
  const size_t rows = (size_t)p.B * p.H * p.L;
  if (pass == 0 && tc_fwd_supported(p)) {
    w.part_off = off;
    off = align_up(off + tc_fwd_part_bytes(p), 256);
    w.qplan_off = off;
    off = align_up(off + tc_qplan_bytes(p), 256);
    w.tdead_off = off;
    off = align_up(off + (size_t)p.B * tc_tdead_words(p) * sizeof(uint32_t), 256);
    w.total = off;
    return w;
  }
  if (pass == 1) {
    w.D_off = off;
    off = align_up(off + rows * sizeof(float), 256);
    w.offs_off = off;
    off = align_up(off + (size_t)p.H * (p.nb + 1) * sizeof(int), 256);
    w.list_off = off;
    off = align_up(off + (size_t)p.H * pair_cap(p.nb, p.r) * sizeof(int), 256);
    if (tc_bwd_supported(p)) {
      w.part_off = off;
      off = align_up(off + tc_bwd_extra_bytes(p), 256);
      w.qplan_off = off;
      off = align_up(off + tc_qplan_bytes(p), 256);
      w.kof_off = off;
      off = align_up(off + ((size_t)p.H * tc_key_items_per_bh(p) * 2 + p.H) * sizeof(int), 256);
      w.kplan_off = off;
      off = align_up(off + (size_t)p.H * tc_kplan_cap(p) * sizeof(uint32_t), 256);
      w.tdead_off = off;
      off = align_up(off + (size_t)p.B * tc_tdead_words(p) * sizeof(uint32_t), 256);
      w.total = off;
      return w;
    }
  }
  w.part_off = off;
  w.total = off;
  return w;
}

}  // namespace bb

using namespace bb;

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kMix1 = 0xBF58476D1CE4E5B9ull;
constexpr uint64_t kMix2 = 0x94D049BB133111EBull;

// SplitMix64 (Steele, Lea and Flood, OOPSLA 2014): add the golden gamma to
// the state, then the two xor-shift-multiply rounds and a final xor-shift.
struct SplitMix64 {
  uint64_t s;
  uint64_t next() {
    s += kGamma;
    uint64_t z = s;
    z = (z ^ (z >> 30)) * kMix1;
    z = (z ^ (z >> 27)) * kMix2;
    return z ^ (z >> 31);
  }
};

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Checks the descriptor and fills the size part of a Problem.
int make_problem(const bb_attn_desc* desc, Problem* p) {
  if (!desc) return BB_ERR_INVALID;
  memset(p, 0, sizeof(*p));
  p->B = desc->B;
  p->H = desc->H;
  p->L = desc->L;
  p->d = desc->d;
  p->bs = desc->block_size;
  p->r = desc->r;
  p->dtype = desc->dtype;
  if (p->B <= 0 || p->H <= 0 || p->L <= 0 || p->d <= 0 || p->bs <= 0 ||
      p->r < 0)
    return BB_ERR_INVALID;
  if (p->dtype != BB_F32 && p->dtype != BB_BF16) return BB_ERR_INVALID;
  if (p->L % p->bs != 0) return BB_ERR_INVALID;
  if (!isfinite(desc->scale) || !isfinite(desc->mask_value))
    return BB_ERR_INVALID;
  // Dropout rate in [0, 1), rounded to 1/256; a rate that rounds to 1 would
  // drop everything (infinite scale).
  if (!(desc->dropout >= 0.f && desc->dropout < 1.f)) return BB_ERR_INVALID;
  const double thr = floor((double)desc->dropout * 256.0 + 0.5);
  if (thr > 255.0) return BB_ERR_INVALID;
  if (p->d != kHeadDim) return BB_ERR_UNSUPPORTED;
  if (p->bs != 32 && p->bs != 64 && p->bs != 128) return BB_ERR_UNSUPPORTED;
  p->nb = p->L / p->bs;
  if (p->nb > kMaxBlocks || p->r > kMaxRand) return BB_ERR_UNSUPPORTED;
  if (p->H > 65535 || p->B > 65535) return BB_ERR_UNSUPPORTED;
  p->scale = desc->scale != 0.f ? desc->scale : 1.0f / sqrtf((float)p->d);
  p->mask_value = desc->mask_value != 0.f ? desc->mask_value : -10000.0f;
  p->drop_thr = (uint32_t)thr;
  p->drop_scale = (float)(256.0 / (256.0 - thr));
  p->drop_seed = desc->dropout_seed;
  if (desc->mask_queries != 0 && desc->mask_queries != 1) return BB_ERR_INVALID;
  p->mask_q = desc->mask_queries;  // cleared at the call when key_mask is NULL
  if (desc->grad_fp32 != 0 && desc->grad_fp32 != 1) return BB_ERR_INVALID;
  p->grad_f32 = (p->dtype == BB_F32) ? 1 : desc->grad_fp32;
  // Stored keep decisions: only with dropout on, and only where both passes
  // run the tensor-core kernels (the one place they are written and read).
  if (desc->dropout_bits && !aligned16(desc->dropout_bits)) return BB_ERR_INVALID;
  if (desc->dropout_bits && p->drop_thr && tc_fwd_supported(*p) && tc_bwd_supported(*p)) {
    p->keep_bits = static_cast<uint32_t*>(desc->dropout_bits);
    p->keep_slots = keep_slots_per_bh(p->nb, p->r);
  }
  return BB_OK;
}

int carve(Problem* p, int pass, void* ws, size_t ws_bytes) {
  if (!ws) return BB_ERR_WORKSPACE;
  if (!aligned16(ws)) return BB_ERR_INVALID;
  WsLayout w = ws_layout(*p, pass);
  if (ws_bytes < w.total) return BB_ERR_WORKSPACE;
  char* base = (char*)ws;
  p->status = (int*)(base + w.status_off);
  p->sched = (int*)(base + w.status_off + 64);  // same 256-byte region
  if (pass == 1) {
    p->D = (float*)(base + w.D_off);
    p->csr_offs = (int*)(base + w.offs_off);
    p->csr_list = (int*)(base + w.list_off);
    p->csr_cap = pair_cap(p->nb, p->r);
  }
  p->part = (float*)(base + w.part_off);
  p->part_floats = (ws_bytes - w.part_off) / sizeof(float);
  if (w.qplan_off) p->qplan = base + w.qplan_off;
  if (w.tdead_off) {
    p->tdead = (uint32_t*)(base + w.tdead_off);
    p->tdead_words = tc_tdead_words(*p);
  }
  if (w.kof_off) {
    p->kof = (int*)(base + w.kof_off);
    p->kplan = (uint32_t*)(base + w.kplan_off);
    p->kcap = tc_kplan_cap(*p);
  }
  return BB_OK;
}

}  // namespace

extern "C" {

int bb_abi_version(void) { return BB_ABI_VERSION; }

const char* bb_status_str(int status) {
  switch (status) {
    case BB_OK: return "ok";
    case BB_ERR_INVALID: return "invalid argument";
    case BB_ERR_UNSUPPORTED: return "unsupported problem size";
    case BB_ERR_CUDA: return "CUDA runtime error";
    case BB_ERR_WORKSPACE: return "workspace missing or too small";
    case BB_ERR_TIMEOUT: return "a device wait ran out of iterations";
    case BB_ERR_BAD_TABLE: return "random table entry out of range (ignored)";
    default: return "unknown status";
  }
}

int bb_rand_attn_build_ex(uint64_t seed, int heads, int num_blocks, int r,
                          int max_blocks, int last_block, int32_t* out_host) {
  if (heads < 0 || num_blocks < 0 || r < 0 || max_blocks < 0 || last_block < 0)
    return BB_ERR_INVALID;
  // The rows are drawn as for a table of nbb blocks; the first num_blocks
  // rows are kept.
  const int nbb = max_blocks ? max_blocks : num_blocks;
  if (nbb < num_blocks) return BB_ERR_INVALID;
  const size_t n = (size_t)heads * num_blocks * r;
  if (n == 0) return BB_OK;
  if (!out_host) return BB_ERR_INVALID;
  std::vector<int32_t> cand;
  cand.reserve(nbb);
  for (int h = 0; h < heads; ++h) {
    for (int i = 0; i < num_blocks; ++i) {
      int32_t* row = out_host + ((size_t)h * num_blocks + i) * r;
      for (int a = 0; a < r; ++a) row[a] = -1;
      if (i == 0 || i == num_blocks - 1) continue;
      cand.clear();
      for (int j = 1; j <= nbb - 2; ++j)
        if ((j < i - 1 || j > i + 1) && (last_block == 0 || j < last_block))
          cand.push_back(j);
      const int m = (int)cand.size();
      const int r_eff = r < m ? r : m;
      SplitMix64 g{seed ^ (((uint64_t)(uint32_t)h << 32) | (uint64_t)(uint32_t)i)};
      for (int a = 0; a < r_eff; ++a) {
        const uint64_t u = g.next();
        const int t = a + (int)(u % (uint64_t)(m - a));
        std::swap(cand[a], cand[t]);
      }
      // Keep the ids of this table's middle blocks: one at or past its last
      // (global) block is dropped, which leaves the attended set unchanged
      // or removes a block the shorter sequence does not have.
      int k = 0;
      for (int a = 0; a < r_eff; ++a)
        if (cand[a] <= num_blocks - 2) row[k++] = cand[a];
      std::sort(row, row + k);
    }
  }
  return BB_OK;
}

int bb_rand_attn_build(uint64_t seed, int heads, int num_blocks, int r,
                       int32_t* out_host) {
  return bb_rand_attn_build_ex(seed, heads, num_blocks, r, 0, 0, out_host);
}

int bb_attn_dropout_bits_size(const bb_attn_desc* desc, size_t* bytes) {
  if (!bytes) return BB_ERR_INVALID;
  Problem p;
  int st = make_problem(desc, &p);
  if (st != BB_OK) return st;
  *bytes = p.drop_thr ? (size_t)p.B * p.H * keep_slots_per_bh(p.nb, p.r) *
                            ((size_t)p.bs * p.bs / 8)
                      : 0;
  return BB_OK;
}

int bb_attn_workspace_size(const bb_attn_desc* desc, int pass, size_t* bytes) {
  if (!bytes || (pass != 0 && pass != 1)) return BB_ERR_INVALID;
  Problem p;
  int st = make_problem(desc, &p);
  if (st != BB_OK) return st;
  *bytes = ws_layout(p, pass).total;
  return BB_OK;
}

static int fwd_impl(const bb_attn_desc* desc, const void* q, const void* k,
                    const void* v, const uint8_t* key_mask,
                    const int32_t* rand_idx, void* out, float* lse,
                    void* workspace, size_t workspace_bytes, void* stream,
                    EventMarks* marks) {
  Problem p;
  int st = make_problem(desc, &p);
  if (st != BB_OK) return st;
  if (!q || !k || !v || !out || !lse) return BB_ERR_INVALID;
  if (p.r > 0 && !rand_idx) return BB_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      !aligned16(lse) || !aligned16(rand_idx) || !aligned16(key_mask))
    return BB_ERR_INVALID;
  st = carve(&p, 0, workspace, workspace_bytes);
  if (st != BB_OK) return st;
  p.q = q;
  p.k = k;
  p.v = v;
  p.key_mask = key_mask;
  if (!key_mask) p.mask_q = 0;
  p.rand_idx = rand_idx;
  p.out = out;
  p.lse_out = lse;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(p.status, 0, sizeof(int), s) != cudaSuccess)
    return BB_ERR_CUDA;
  if (marks->mark(s) != cudaSuccess) return BB_ERR_CUDA;
  if (tc_fwd_supported(p)) {
    TensorMaps tm;
    if (!encode_tensor_maps(p, 0, &tm)) return BB_ERR_CUDA;
    if (launch_plan(p, false, s) != cudaSuccess) return BB_ERR_CUDA;
    if (marks->mark(s) != cudaSuccess) return BB_ERR_CUDA;
    if (launch_tc_fwd(p, tm, s, marks) != cudaSuccess) return BB_ERR_CUDA;
  } else {
    if (launch_simt_fwd(p, s) != cudaSuccess) return BB_ERR_CUDA;
  }
  if (marks->mark(s) != cudaSuccess) return BB_ERR_CUDA;
  return BB_OK;
}

static int bwd_impl(const bb_attn_desc* desc, const void* q, const void* k,
                    const void* v, const void* out, const float* lse,
                    const void* dout, const uint8_t* key_mask,
                    const int32_t* rand_idx, void* dq, void* dk, void* dv,
                    void* workspace, size_t workspace_bytes, void* stream,
                    EventMarks* marks) {
  Problem p;
  int st = make_problem(desc, &p);
  if (st != BB_OK) return st;
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv)
    return BB_ERR_INVALID;
  if (p.r > 0 && !rand_idx) return BB_ERR_INVALID;
  const void* ptrs[] = {q, k, v, out, lse, dout, key_mask, rand_idx,
                        dq, dk, dv};
  for (const void* x : ptrs)
    if (!aligned16(x)) return BB_ERR_INVALID;
  st = carve(&p, 1, workspace, workspace_bytes);
  if (st != BB_OK) return st;
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = out;
  p.lse = lse;
  p.dout = dout;
  p.key_mask = key_mask;
  if (!key_mask) p.mask_q = 0;
  p.rand_idx = rand_idx;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(p.status, 0, sizeof(int), s) != cudaSuccess)
    return BB_ERR_CUDA;
  if (marks->mark(s) != cudaSuccess) return BB_ERR_CUDA;
  if (tc_bwd_supported(p)) {
    TensorMaps tm;
    if (!encode_tensor_maps(p, 1, &tm)) return BB_ERR_CUDA;
    if (tc_bwd_plan_fused(p)) {
      if (launch_plan_bwd(p, s) != cudaSuccess) return BB_ERR_CUDA;
    } else {
      if (launch_csr_build(p, s) != cudaSuccess) return BB_ERR_CUDA;
      if (marks->mark(s) != cudaSuccess) return BB_ERR_CUDA;
      if (launch_plan(p, true, s) != cudaSuccess) return BB_ERR_CUDA;
    }
    if (marks->mark(s) != cudaSuccess) return BB_ERR_CUDA;
    if (launch_tc_bwd(p, tm, s, marks) != cudaSuccess) return BB_ERR_CUDA;
  } else {
    if (launch_bwd_pre(p, s) != cudaSuccess) return BB_ERR_CUDA;
    if (marks->mark(s) != cudaSuccess) return BB_ERR_CUDA;
    if (launch_csr_build(p, s) != cudaSuccess) return BB_ERR_CUDA;
    if (marks->mark(s) != cudaSuccess) return BB_ERR_CUDA;
    if (launch_simt_bwd(p, s, marks) != cudaSuccess) return BB_ERR_CUDA;
  }
  if (marks->mark(s) != cudaSuccess) return BB_ERR_CUDA;
  return BB_OK;
}

// Names of the launches each pass makes, in order (kept beside the
// dispatch in fwd_impl / bwd_impl).
static const char* const kFwdSimt[] = {"simt_fwd"};
static const char* const kFwdTc[] = {"plan", "tc_fwd", "fwd_combine"};
static const char* const kBwdSimt[] = {"bwd_pre", "csr_build", "simt_dq",
                                       "simt_dkdv"};
// Tensor-core backward: the plans (with each head's transposed adjacency
// built in shared memory, one launch) or, when a head's adjacency does not
// fit there, csr_build + plan; then dQ, dK/dV (two launches at long lengths:
// the global key blocks with the hi/lo split on their own,
// tc_dkdv_launches), and the merge of the global rows' partials when those
// rows are split into chunks (tc_global_rows_chunked; the forward's
// fwd_combine likewise).
static const char* const kBwdTcTail1[] = {"tc_dq", "tc_dkdv", "bwd_finish"};
static const char* const kBwdTcTail2[] = {"tc_dq", "tc_dkdv", "tc_dkdv", "bwd_finish"};

static int launch_plan(const bb_attn_desc* desc, int pass,
                       const char* const** names, int* n) {
  if (pass != 0 && pass != 1) return BB_ERR_INVALID;
  Problem p;
  int st = make_problem(desc, &p);
  if (st != BB_OK) return st;
  if (pass == 0) {
    const bool tc = tc_fwd_supported(p);
    *names = tc ? kFwdTc : kFwdSimt;
    *n = tc ? (tc_global_rows_chunked(p, 0) ? 3 : 2) : 1;
  } else {
    if (!tc_bwd_supported(p)) {
      *names = kBwdSimt;
      *n = 4;
      return BB_OK;
    }
    // Assembled per shape in a small table owned by this translation unit.
    static thread_local const char* buf[8];
    int c = 0;
    if (!tc_bwd_plan_fused(p)) buf[c++] = "csr_build";
    buf[c++] = "plan";
    const bool two = tc_dkdv_launches(p) == 2;
    const char* const* tail = two ? kBwdTcTail2 : kBwdTcTail1;
    // The merge launch only when global rows are chunked.
    const int nt = (two ? 4 : 3) - (tc_global_rows_chunked(p, 1) ? 0 : 1);
    for (int i = 0; i < nt; ++i) buf[c++] = tail[i];
    *names = buf;
    *n = c;
  }
  return BB_OK;
}

int bb_attn_launch_count(const bb_attn_desc* desc, int pass, int* launches) {
  if (!launches) return BB_ERR_INVALID;
  const char* const* names;
  return launch_plan(desc, pass, &names, launches);
}

int bb_attn_launch_name(const bb_attn_desc* desc, int pass, int index,
                        const char** name) {
  if (!name) return BB_ERR_INVALID;
  const char* const* names;
  int n = 0;
  int st = launch_plan(desc, pass, &names, &n);
  if (st != BB_OK) return st;
  if (index < 0 || index >= n) return BB_ERR_INVALID;
  *name = names[index];
  return BB_OK;
}

int bb_attn_fwd(const bb_attn_desc* desc, const void* q, const void* k,
                const void* v, const uint8_t* key_mask,
                const int32_t* rand_idx, void* out, float* lse,
                void* workspace, size_t workspace_bytes, void* stream) {
  EventMarks m;
  return fwd_impl(desc, q, k, v, key_mask, rand_idx, out, lse, workspace,
                  workspace_bytes, stream, &m);
}

int bb_attn_fwd_events(const bb_attn_desc* desc, const void* q,
                       const void* k, const void* v, const uint8_t* key_mask,
                       const int32_t* rand_idx, void* out, float* lse,
                       void* workspace, size_t workspace_bytes, void* stream,
                       void* const* events, int num_events) {
  EventMarks m;
  m.ev = events;
  m.n = num_events;
  return fwd_impl(desc, q, k, v, key_mask, rand_idx, out, lse, workspace,
                  workspace_bytes, stream, &m);
}

int bb_attn_bwd(const bb_attn_desc* desc, const void* q, const void* k,
                const void* v, const void* out, const float* lse,
                const void* dout, const uint8_t* key_mask,
                const int32_t* rand_idx, void* dq, void* dk, void* dv,
                void* workspace, size_t workspace_bytes, void* stream) {
  EventMarks m;
  return bwd_impl(desc, q, k, v, out, lse, dout, key_mask, rand_idx, dq, dk,
                  dv, workspace, workspace_bytes, stream, &m);
}

int bb_attn_bwd_events(const bb_attn_desc* desc, const void* q,
                       const void* k, const void* v, const void* out,
                       const float* lse, const void* dout,
                       const uint8_t* key_mask, const int32_t* rand_idx,
                       void* dq, void* dk, void* dv, void* workspace,
                       size_t workspace_bytes, void* stream,
                       void* const* events, int num_events) {
  EventMarks m;
  m.ev = events;
  m.n = num_events;
  return bwd_impl(desc, q, k, v, out, lse, dout, key_mask, rand_idx, dq, dk,
                  dv, workspace, workspace_bytes, stream, &m);
}

int bb_attn_check_status(const void* workspace, void* stream) {
  if (!workspace) return BB_ERR_INVALID;
  int h = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return BB_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BB_ERR_CUDA;
  return h;
}

}  // extern "C"
