// C ABI of the LISA layer: host-side validation, workspace carve-up, launches.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <unordered_map>

#include "lisa_internal.h"

namespace {

thread_local char g_msg[512] = "";

lisa_status fail(lisa_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

lisa_status ok() {
  g_msg[0] = '\0';
  return LISA_OK;
}

lisa_status cuda_fail(cudaError_t e, const char *where) {
  return fail(LISA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

int round4(int x) { return (x + 3) & ~3; }

constexpr int kRowsStagedCap = 2048;   // keys of a row staged in shared memory by the row select
constexpr int kCandCap = 2048;          // threshold-bucket candidates kept in shared memory (a small
                                        // footprint lets about six select CTAs share an SM)
constexpr int kRowChunk = 2048;         // query rows scored per pass on the row path
constexpr int kMaxSmem = 227 * 1024;    // dynamic shared memory a CTA may use on sm_100

// Validates the geometry; returns LISA_OK or the failure status.
lisa_status check_layer(const lisa_layer *L) {
  if (!L) return fail(LISA_ERR_INVALID_ARG, "layer is NULL");
  if (L->B < 0 || L->Hq < 1 || L->Hkv < 1 || L->HI < 1 || L->d < 1 || L->dI < 1 || L->M < 1 || L->L_max < 1)
    return fail(LISA_ERR_INVALID_ARG, "non-positive dimension (B=%d Hq=%d Hkv=%d HI=%d d=%d dI=%d M=%d L_max=%d)",
                L->B, L->Hq, L->Hkv, L->HI, L->d, L->dI, L->M, L->L_max);
  if (L->dtype != LISA_BF16 && L->dtype != LISA_FP32) return fail(LISA_ERR_INVALID_ARG, "unknown dtype %d", L->dtype);
  if (L->Hq % L->Hkv) return fail(LISA_ERR_UNSUPPORTED, "Hq=%d is not a multiple of Hkv=%d", L->Hq, L->Hkv);
  if (L->HI % L->Hkv) return fail(LISA_ERR_UNSUPPORTED, "HI=%d is not a multiple of Hkv=%d", L->HI, L->Hkv);
  if (L->Hq / L->Hkv > lisa::kMaxG) return fail(LISA_ERR_UNSUPPORTED, "Hq/Hkv=%d > %d", L->Hq / L->Hkv, lisa::kMaxG);
  if (L->HI / L->Hkv > lisa::kMaxR) return fail(LISA_ERR_UNSUPPORTED, "HI/Hkv=%d > %d", L->HI / L->Hkv, lisa::kMaxR);
  if (L->d != 64 && L->d != 128) return fail(LISA_ERR_UNSUPPORTED, "d=%d not in {64,128}", L->d);
  if (L->dI != 32 && L->dI != 64) return fail(LISA_ERR_UNSUPPORTED, "dI=%d not in {32,64}", L->dI);
  if (L->M % 32 || L->M < 32 || L->M > 1024) return fail(LISA_ERR_UNSUPPORTED, "M=%d not a multiple of 32 in [32,1024]", L->M);
  if ((long long)L->B * L->Hkv > 65535) return fail(LISA_ERR_UNSUPPORTED, "B*Hkv=%lld > 65535", (long long)L->B * L->Hkv);
  if (L->decode_split != 0 && L->decode_split != 4 && L->decode_split != 8 && L->decode_split != 16 &&
      L->decode_split != 32 && L->decode_split != 64)
    return fail(LISA_ERR_INVALID_ARG, "decode_split=%d not in {0, 4, 8, 16, 32, 64}", L->decode_split);
  return LISA_OK;
}

lisa_status check_ptr(const void *p, const char *name, bool required = true) {
  if (!p) return required ? fail(LISA_ERR_INVALID_ARG, "%s is NULL", name) : LISA_OK;
  if (!aligned16(p)) return fail(LISA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return LISA_OK;
}

lisa_status check_caches(const lisa_layer *L) {
  lisa_status s;
  if ((s = check_ptr(L->k_cache, "k_cache"))) return s;
  if ((s = check_ptr(L->v_cache, "v_cache"))) return s;
  if ((s = check_ptr(L->kidx_cache, "kidx_cache"))) return s;
  if ((s = check_ptr(L->pos, "pos"))) return s;
  if (L->err_word && (reinterpret_cast<uintptr_t>(L->err_word) & 3u)) return fail(LISA_ERR_INVALID_ARG, "err_word misaligned");
  return LISA_OK;
}

// ---------------------------------------------------------------- workspace plans
struct RowsPlan {
  int row_chunk, L_keys;
  size_t keys, idx, olin, dS, Ptot, total;
};
RowsPlan rows_plan(const lisa_layer *L, int T, bool prefill, bool indexer = true) {
  RowsPlan p;
  const size_t BH = (size_t)L->B * L->Hkv;
  p.row_chunk = T < kRowChunk ? T : kRowChunk;
  p.L_keys = round4(prefill ? T : L->L_max);
  size_t off = 0;
  p.keys = off; off += indexer ? round256(BH * p.row_chunk * p.L_keys * 4) : 0;
  p.idx = p.olin = p.dS = p.Ptot = 0;
  if (prefill) {
    const size_t nc = (T + lisa::kLinChunk - 1) / lisa::kLinChunk;
    p.idx = off; off += round256((size_t)L->B * T * L->Hkv * L->M * 4);
    p.olin = off; off += round256((size_t)L->B * T * L->Hq * L->d * 4);
    p.dS = off; off += round256(BH * nc * L->d * L->d * 4);
    p.Ptot = off; off += round256(BH * L->d * L->d * 4);
  }
  p.total = off;
  return p;
}

void fill_rows(lisa::RowsParams &r, const lisa_layer *L, int T) {
  memset(&r, 0, sizeof(r));
  r.B = L->B; r.Hq = L->Hq; r.Hkv = L->Hkv; r.G = L->Hq / L->Hkv; r.HI = L->HI; r.R = L->HI / L->Hkv;
  r.D = L->d; r.DI = L->dI; r.M = L->M; r.L_max = L->L_max; r.T = T;
  r.scale = (float)(1.0 / sqrt((double)L->d));
  r.k_cache = L->k_cache; r.v_cache = L->v_cache; r.kidx_cache = L->kidx_cache;
  r.state = L->state; r.pos = L->pos; r.err_word = L->err_word;
  r.sel_heads = L->Hkv;
}

// ---------------------------------------------------------------- definition variants
// Geometry of a variant: P indexer-key planes, Gs selection groups.
struct VariantGeom {
  bool per_head, shared, lin_kv;
  int P, Gs;
  bool row_indexer() const { return per_head || shared; }   // indexer + top-M through the row path
};

lisa_status check_variant(const lisa_layer *L, int variant, VariantGeom &vg) {
  if (variant & ~(LISA_VAR_KEY_PER_INDEXER_HEAD | LISA_VAR_SHARED_SET | LISA_VAR_LINEAR_KV_PER_QUERY_HEAD))
    return fail(LISA_ERR_INVALID_ARG, "unknown variant bits 0x%x", variant);
  vg.per_head = (variant & LISA_VAR_KEY_PER_INDEXER_HEAD) != 0;
  vg.shared = (variant & LISA_VAR_SHARED_SET) != 0;
  vg.lin_kv = (variant & LISA_VAR_LINEAR_KV_PER_QUERY_HEAD) != 0;
  vg.Gs = vg.shared ? 1 : L->Hkv;
  vg.P = vg.per_head ? L->HI : vg.Gs;
  if (!vg.per_head && L->HI / vg.Gs > lisa::kMaxR)
    return fail(LISA_ERR_UNSUPPORTED, "%d indexer heads per selection group > %d", L->HI / vg.Gs, lisa::kMaxR);
  return LISA_OK;
}

struct VarPlan {
  int row_chunk, L_keys;
  size_t keys, keys_h, idx, olin, dS, Ptot, total;
};
// op: LISA_OP_DECODE (T = 1 row at pos[b]), LISA_OP_INDEXER_TOPK or LISA_OP_PREFILL.
VarPlan var_plan(const lisa_layer *L, const VariantGeom &vg, int T, int op) {
  VarPlan p;
  memset(&p, 0, sizeof(p));
  const bool prefill = op == LISA_OP_PREFILL;
  const bool indexer = op == LISA_OP_INDEXER_TOPK || prefill || vg.row_indexer();
  if (op == LISA_OP_DECODE) T = 1;
  p.row_chunk = T < kRowChunk ? T : kRowChunk;
  p.L_keys = round4(prefill ? T : L->L_max);
  const size_t rk = (size_t)p.row_chunk * p.L_keys * 4;
  size_t off = 0;
  if (indexer) {
    p.keys = off; off += round256((size_t)L->B * vg.Gs * rk);
    if (vg.P != vg.Gs) { p.keys_h = off; off += round256((size_t)L->B * L->HI * rk); }
  }
  if (prefill || (op == LISA_OP_DECODE && vg.row_indexer())) {
    p.idx = off; off += round256((size_t)L->B * T * vg.Gs * L->M * 4);
  }
  if (prefill) {
    const size_t LH = vg.lin_kv ? L->Hq : L->Hkv;
    const size_t nc = (T + lisa::kLinChunk - 1) / lisa::kLinChunk;
    p.olin = off; off += round256((size_t)L->B * T * L->Hq * L->d * 4);
    p.dS = off; off += round256((size_t)L->B * LH * nc * L->d * L->d * 4);
    p.Ptot = off; off += round256((size_t)L->B * LH * L->d * L->d * 4);
  }
  p.total = off;
  return p;
}

void set_select_smem(lisa::RowsParams &r, int n_max);

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 148;
  }
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;
    }
    cache[dev] = n;
  }
  return cache[dev];
}

// Workspace of lisa_decode_step: that of the wide form (bf16), sized for 64
// CTAs per (sequence, KV head); 0 for fp32 storage.
size_t decode_workspace_bytes(const lisa_layer *L) {
  if (L->dtype != LISA_BF16) return 0;
  return lisa::decode_wide_workspace_bytes(L->B, L->Hkv, L->Hq / L->Hkv, L->d, L->L_max, 64);
}

// Picks the decode form.  The wide form (decode_split 32 or 64, or the
// library's choice when the workspace is given and few (sequence, KV head)
// pairs leave SMs idle) needs bf16 storage and the decode workspace; its
// pieces are carved out of the workspace here.
lisa_status plan_decode_form(const lisa_layer *L, void *workspace, size_t ws_bytes, lisa::DecodeParams &p) {
  const int G = L->Hq / L->Hkv;
  const size_t need = decode_workspace_bytes(L);
  const bool explicit_wide = L->decode_split == 32 || L->decode_split == 64;
  int nw = 0;
  if (explicit_wide) {
    if (L->dtype != LISA_BF16)
      return fail(LISA_ERR_UNSUPPORTED, "decode_split=%d (the wide form) needs bf16 storage", L->decode_split);
    if (L->decode_split < G)
      return fail(LISA_ERR_UNSUPPORTED, "decode_split=%d is smaller than Hq/Hkv=%d", L->decode_split, G);
    if (!workspace || ws_bytes < need)
      return fail(LISA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace ? ws_bytes : 0, need);
    nw = L->decode_split;
  } else if (L->decode_split == 0 && need && workspace && ws_bytes >= need) {
    nw = lisa::decode_wide_nw(L->B, L->Hkv, G, L->d, L->dI, L->dtype, sm_count());
  }
  if (nw && lisa::decode_wide_smem_bytes(L->L_max, L->M, G, L->d, L->dI, nw) > kMaxSmem) {
    if (explicit_wide)
      return fail(LISA_ERR_UNSUPPORTED, "L_max=%d needs more shared memory per CTA than a B200 SM has", L->L_max);
    nw = 0;
  }
  if (!nw) return LISA_OK;
  lisa_status s;
  if ((s = check_ptr(workspace, "workspace"))) return s;
  const size_t pairs = (size_t)L->B * L->Hkv;
  char *ws = static_cast<char *>(workspace);
  size_t off = 0;
  p.wcount = reinterpret_cast<unsigned *>(ws + off); off += round256(pairs * 4);
  p.wpart = reinterpret_cast<float *>(ws + off); off += round256(pairs * 64 * 2 * L->d * 4);
  p.wkeys = reinterpret_cast<uint32_t *>(ws + off);
  p.wkeys_stride = round4(L->L_max);
  p.nw = nw;
  return LISA_OK;
}

// Row-path parameters of the variant's indexer: `sel` scores and selects in
// the Gs selection groups; with one key per indexer head, `ph` first scores
// every indexer head on its own (the groups' sums are formed afterwards).
void variant_indexer_params(const lisa_layer *L, const VariantGeom &vg, int T, const VarPlan &plan, char *ws,
                            const void *qidx, const float *w, int *idx, int n_max, lisa::RowsParams &sel,
                            lisa::RowsParams &ph) {
  fill_rows(sel, L, T);
  sel.Hkv = vg.Gs; sel.R = L->HI / vg.Gs; sel.G = L->Hq / vg.Gs; sel.sel_heads = vg.Gs;
  sel.qidx = qidx; sel.w = w; sel.idx = idx;
  sel.keys = reinterpret_cast<uint32_t *>(ws + plan.keys);
  sel.row_chunk = plan.row_chunk;
  sel.L_keys = plan.L_keys;
  set_select_smem(sel, n_max);
  ph = sel;
  ph.Hkv = L->HI; ph.R = 1; ph.G = 1; ph.sel_heads = L->HI;
  ph.keys = vg.P != vg.Gs ? reinterpret_cast<uint32_t *>(ws + plan.keys_h) : nullptr;
}

// Appends the indexer keys of T tokens ([B, T, P, dI]) at pos[b] + tau.
cudaError_t append_kidx_planes(const lisa_layer *L, const VariantGeom &vg, int T, const void *kidx, int require_pos0,
                               cudaStream_t st) {
  lisa::RowsParams a;
  fill_rows(a, L, T);
  a.Hkv = vg.P; a.R = 1; a.G = 1;
  a.require_pos0 = require_pos0;
  a.kidx = kidx;
  return lisa::launch_append(a, L->dtype, st);
}

void set_select_smem(lisa::RowsParams &r, int n_max) {
  // rows of up to 2048 keys are staged in shared memory; longer rows are read
  // from global memory by the bounded select
  const int cap = n_max < kRowsStagedCap ? n_max : kRowsStagedCap;
  r.smem_keys_cap = (cap + 3) & ~3;
  r.cand_cap = kCandCap;
  r.select_smem = (size_t)(r.smem_keys_cap + 2 * r.cand_cap) * 4;   // keys, candidate keys and positions
}

}  // namespace

namespace lisa {

cudaError_t prepare_kernel_ptr(const void *fn, int dyn_smem) {
  static std::mutex mu;
  static std::unordered_map<const void *, int> done[64];   // per device: kernel -> dynamic smem limit set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto &m = done[dev & 63];
  auto it = m.find(fn);
  if (it == m.end()) it = m.emplace(fn, 0).first;
  if (dyn_smem > it->second) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_smem);
    if (e != cudaSuccess) return e;
    it->second = dyn_smem;
  }
  return cudaSuccess;
}

}  // namespace lisa

// ---------------------------------------------------------------- fixed scratch
// Scratch of lisa_indexer_topk_noalloc(): a fixed array in device memory that
// every GPU loading this library holds until the process exits.  Host code
// must not pass `g_noalloc_scratch` itself to a kernel (on the host that name
// is only a stand-in); it asks the runtime for the array's device address once
// per device, with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LISA_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mu;
void *g_noalloc_addr[64] = {nullptr};

// Device address of g_noalloc_scratch on the current device (looked up on the
// first call for that device, cached afterwards).
lisa_status noalloc_scratch(void **addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LISA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    g_noalloc_addr[dev] = p;
  }
  *addr = g_noalloc_addr[dev];
  return LISA_OK;
}

}  // namespace

extern "C" {

const char *lisa_version(void) { return "lisa-b200 0.1 (sm_100a)"; }

const char *lisa_last_error_msg(void) { return g_msg; }

const char *lisa_status_str(lisa_status s) {
  switch (s) {
    case LISA_OK: return "LISA_OK";
    case LISA_ERR_INVALID_ARG: return "LISA_ERR_INVALID_ARG";
    case LISA_ERR_UNSUPPORTED: return "LISA_ERR_UNSUPPORTED";
    case LISA_ERR_CUDA: return "LISA_ERR_CUDA";
    case LISA_ERR_WORKSPACE: return "LISA_ERR_WORKSPACE";
  }
  return "LISA_ERR_UNKNOWN";
}

size_t lisa_workspace_bytes(const lisa_layer *layer, int T, int op) {
  if (check_layer(layer) != LISA_OK || T < 0) return 0;
  if (op == LISA_OP_DECODE) return decode_workspace_bytes(layer);
  if (op == LISA_OP_PREFILL) return T ? rows_plan(layer, T, true).total : 0;
  if (op == LISA_OP_INDEXER_TOPK) return T ? rows_plan(layer, T, false).total : 0;
  if (op == LISA_OP_PREFILL_WINDOW) return T ? rows_plan(layer, T, true, false).total : 0;
  return 0;
}

lisa_status lisa_append_cache(const lisa_layer *L, const void *k, const void *v, const void *kidx, int T,
                              void *stream) {
  lisa_status s;
  if ((s = check_layer(L))) return s;
  if (T < 0) return fail(LISA_ERR_INVALID_ARG, "T=%d < 0", T);
  if (T == 0 || L->B == 0) return ok();
  if (T > L->L_max) return fail(LISA_ERR_INVALID_ARG, "T=%d > L_max=%d", T, L->L_max);
  if ((s = check_caches(L))) return s;
  if ((s = check_ptr(k, "k")) || (s = check_ptr(v, "v")) || (s = check_ptr(kidx, "kidx"))) return s;
  lisa::RowsParams r;
  fill_rows(r, L, T);
  r.k = k; r.v = v; r.kidx = kidx;
  cudaError_t e = lisa::launch_append(r, L->dtype, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "append");
  return ok();
}

lisa_status lisa_indexer_topk(const lisa_layer *L, const void *qidx, const float *w, int T, int *idx_out,
                              void *workspace, size_t ws_bytes, void *stream) {
  lisa_status s;
  if ((s = check_layer(L))) return s;
  if (T < 0) return fail(LISA_ERR_INVALID_ARG, "T=%d < 0", T);
  if (T == 0 || L->B == 0) return ok();
  if (T > L->L_max) return fail(LISA_ERR_INVALID_ARG, "T=%d > L_max=%d", T, L->L_max);
  if ((s = check_caches(L))) return s;
  if ((s = check_ptr(qidx, "qidx")) || (s = check_ptr(w, "w")) || (s = check_ptr(idx_out, "idx_out"))) return s;
  const RowsPlan plan = rows_plan(L, T, false);
  if (!workspace || ws_bytes < plan.total)
    return fail(LISA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace ? ws_bytes : 0, plan.total);
  if ((s = check_ptr(workspace, "workspace"))) return s;
  lisa::RowsParams r;
  fill_rows(r, L, T);
  r.qidx = qidx; r.w = w; r.idx = idx_out;
  char *ws = static_cast<char *>(workspace);
  r.keys = reinterpret_cast<uint32_t *>(ws + plan.keys);
  r.row_chunk = plan.row_chunk;
  r.L_keys = plan.L_keys;
  set_select_smem(r, L->L_max);
  cudaError_t e = lisa::launch_rows_topk(r, L->dtype, (cudaStream_t)stream, L->L_max);
  if (e != cudaSuccess) return cuda_fail(e, "indexer_topk");
  return ok();
}

lisa_status lisa_decode_step(const lisa_layer *L, const void *q, const void *k, const void *v, const void *kidx,
                             const void *qidx, const float *w, const float *gate_logit, int fuse_append, void *out,
                             int *idx_out, void *workspace, size_t ws_bytes, void *stream) {
  lisa_status s;
  if ((s = check_layer(L))) return s;
  if (L->B == 0) return ok();
  if ((s = check_caches(L))) return s;
  if ((s = check_ptr(L->state, "state"))) return s;
  if ((s = check_ptr(q, "q")) || (s = check_ptr(k, "k")) || (s = check_ptr(v, "v")) || (s = check_ptr(kidx, "kidx")) ||
      (s = check_ptr(qidx, "qidx")) || (s = check_ptr(w, "w")) || (s = check_ptr(gate_logit, "gate_logit")) ||
      (s = check_ptr(out, "out")) || (s = check_ptr(idx_out, "idx_out", false)))
    return s;
  const int esz = L->dtype == LISA_BF16 ? 2 : 4;
  if (lisa::decode_smem_bytes(L->L_max, L->M, L->Hq / L->Hkv, L->d, L->dI, esz, 8) > kMaxSmem)
    return fail(LISA_ERR_UNSUPPORTED, "L_max=%d needs more shared memory per CTA than a B200 SM has", L->L_max);

  lisa::DecodeParams p;
  memset(&p, 0, sizeof(p));
  p.B = L->B; p.Hq = L->Hq; p.Hkv = L->Hkv; p.G = L->Hq / L->Hkv; p.HI = L->HI; p.R = L->HI / L->Hkv;
  p.D = L->d; p.DI = L->dI; p.M = L->M; p.L_max = L->L_max; p.fuse_append = fuse_append ? 1 : 0;
  p.split_req = L->decode_split;
  p.independent = L->independent ? 1 : 0;
  p.debug_flags = L->debug_flags;
  p.scale = (float)(1.0 / sqrt((double)L->d));
  p.k_cache = L->k_cache; p.v_cache = L->v_cache; p.kidx_cache = L->kidx_cache;
  p.state = L->state; p.pos = L->pos; p.err_word = L->err_word;
  p.q = q; p.k = k; p.v = v; p.kidx = kidx; p.qidx = qidx; p.w = w; p.gate = gate_logit;
  p.out = out; p.idx_out = idx_out;
  if ((s = plan_decode_form(L, workspace, ws_bytes, p))) return s;
  cudaError_t e = lisa::launch_decode(p, L->dtype, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode_step");
  return ok();
}

lisa_status lisa_decode_step_window(const lisa_layer *L, const void *q, const void *k, const void *v,
                                    const void *kidx, const float *gate_logit, int fuse_append, void *out,
                                    int *idx_out, void *stream) {
  lisa_status s;
  if ((s = check_layer(L))) return s;
  if (L->B == 0) return ok();
  if ((s = check_caches(L))) return s;
  if ((s = check_ptr(L->state, "state"))) return s;
  if ((s = check_ptr(q, "q")) || (s = check_ptr(k, "k")) || (s = check_ptr(v, "v")) ||
      (s = check_ptr(kidx, "kidx", false)) || (s = check_ptr(gate_logit, "gate_logit")) ||
      (s = check_ptr(out, "out")) || (s = check_ptr(idx_out, "idx_out", false)))
    return s;
  const int esz = L->dtype == LISA_BF16 ? 2 : 4;
  if (lisa::decode_smem_bytes(L->L_max, L->M, L->Hq / L->Hkv, L->d, L->dI, esz, 8) > kMaxSmem)
    return fail(LISA_ERR_UNSUPPORTED, "L_max=%d needs more shared memory per CTA than a B200 SM has", L->L_max);
  lisa::DecodeParams p;
  memset(&p, 0, sizeof(p));
  p.B = L->B; p.Hq = L->Hq; p.Hkv = L->Hkv; p.G = L->Hq / L->Hkv; p.HI = L->HI; p.R = L->HI / L->Hkv;
  p.D = L->d; p.DI = L->dI; p.M = L->M; p.L_max = L->L_max; p.fuse_append = fuse_append ? 1 : 0;
  p.split_req = L->decode_split;
  p.independent = L->independent ? 1 : 0;
  p.debug_flags = L->debug_flags;
  p.window = 1;
  p.scale = (float)(1.0 / sqrt((double)L->d));
  p.k_cache = L->k_cache; p.v_cache = L->v_cache; p.kidx_cache = L->kidx_cache;
  p.state = L->state; p.pos = L->pos; p.err_word = L->err_word;
  p.q = q; p.k = k; p.v = v; p.kidx = kidx; p.qidx = nullptr; p.w = nullptr; p.gate = gate_logit;
  p.out = out; p.idx_out = idx_out;
  cudaError_t e = lisa::launch_decode(p, L->dtype, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode_step_window");
  return ok();
}

lisa_status lisa_prefill_window(const lisa_layer *L, int T, const void *q, const void *k, const void *v,
                                const void *kidx, const float *gate_logit, void *out, int *idx_out, void *workspace,
                                size_t ws_bytes, void *stream) {
  lisa_status s;
  if ((s = check_layer(L))) return s;
  if (T < 0) return fail(LISA_ERR_INVALID_ARG, "T=%d < 0", T);
  if (T == 0 || L->B == 0) return ok();
  if (T > L->L_max) return fail(LISA_ERR_INVALID_ARG, "T=%d > L_max=%d", T, L->L_max);
  if ((s = check_caches(L))) return s;
  if ((s = check_ptr(L->state, "state"))) return s;
  if ((s = check_ptr(q, "q")) || (s = check_ptr(k, "k")) || (s = check_ptr(v, "v")) ||
      (s = check_ptr(kidx, "kidx", false)) || (s = check_ptr(gate_logit, "gate_logit")) ||
      (s = check_ptr(out, "out")) || (s = check_ptr(idx_out, "idx_out", false)))
    return s;
  const RowsPlan plan = rows_plan(L, T, true, false);
  if (!workspace || ws_bytes < plan.total)
    return fail(LISA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace ? ws_bytes : 0, plan.total);
  if ((s = check_ptr(workspace, "workspace"))) return s;

  lisa::RowsParams r;
  fill_rows(r, L, T);
  r.require_pos0 = 1;
  r.q = q; r.k = k; r.v = v; r.kidx = kidx; r.qidx = nullptr; r.w = nullptr; r.gate = gate_logit; r.out = out;
  char *ws = static_cast<char *>(workspace);
  r.keys = nullptr;
  r.idx = idx_out ? idx_out : reinterpret_cast<int *>(ws + plan.idx);
  r.olin = reinterpret_cast<float *>(ws + plan.olin);
  r.dS = reinterpret_cast<float *>(ws + plan.dS);
  r.Ptot = reinterpret_cast<float *>(ws + plan.Ptot);
  r.row_chunk = plan.row_chunk;
  r.L_keys = plan.L_keys;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = lisa::launch_append(r, L->dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill_window append");
  e = lisa::launch_prefill_linear(r, L->dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill_window linear");
  e = lisa::launch_window_idx(r, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill_window index");
  e = lisa::launch_prefill_attend(r, L->dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill_window attend");
  return ok();
}

lisa_status lisa_prefill(const lisa_layer *L, int T, const void *q, const void *k, const void *v, const void *kidx,
                         const void *qidx, const float *w, const float *gate_logit, void *out, int *idx_out,
                         void *workspace, size_t ws_bytes, void *stream) {
  lisa_status s;
  if ((s = check_layer(L))) return s;
  if (T < 0) return fail(LISA_ERR_INVALID_ARG, "T=%d < 0", T);
  if (T == 0 || L->B == 0) return ok();
  if (T > L->L_max) return fail(LISA_ERR_INVALID_ARG, "T=%d > L_max=%d", T, L->L_max);
  if ((s = check_caches(L))) return s;
  if ((s = check_ptr(L->state, "state"))) return s;
  if ((s = check_ptr(q, "q")) || (s = check_ptr(k, "k")) || (s = check_ptr(v, "v")) || (s = check_ptr(kidx, "kidx")) ||
      (s = check_ptr(qidx, "qidx")) || (s = check_ptr(w, "w")) || (s = check_ptr(gate_logit, "gate_logit")) ||
      (s = check_ptr(out, "out")) || (s = check_ptr(idx_out, "idx_out", false)))
    return s;
  const RowsPlan plan = rows_plan(L, T, true);
  if (!workspace || ws_bytes < plan.total)
    return fail(LISA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace ? ws_bytes : 0, plan.total);
  if ((s = check_ptr(workspace, "workspace"))) return s;

  lisa::RowsParams r;
  fill_rows(r, L, T);
  r.require_pos0 = 1;
  r.q = q; r.k = k; r.v = v; r.kidx = kidx; r.qidx = qidx; r.w = w; r.gate = gate_logit; r.out = out;
  char *ws = static_cast<char *>(workspace);
  r.idx = idx_out ? idx_out : reinterpret_cast<int *>(ws + plan.idx);
  r.olin = reinterpret_cast<float *>(ws + plan.olin);
  r.dS = reinterpret_cast<float *>(ws + plan.dS);
  r.Ptot = reinterpret_cast<float *>(ws + plan.Ptot);
  r.keys = reinterpret_cast<uint32_t *>(ws + plan.keys);
  r.row_chunk = plan.row_chunk;
  r.L_keys = plan.L_keys;
  set_select_smem(r, T);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = lisa::launch_append(r, L->dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill append");
  e = lisa::launch_prefill_linear(r, L->dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill linear");
  e = lisa::launch_rows_topk(r, L->dtype, st, T);
  if (e != cudaSuccess) return cuda_fail(e, "prefill indexer");
  e = lisa::launch_prefill_attend(r, L->dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill attend");
  return ok();
}

lisa_status lisa_indexer_kl(const lisa_layer *L, int T, const void *q, const void *qidx, const float *w, float *kl_out,
                            void *stream) {
  lisa_status s;
  if ((s = check_layer(L))) return s;
  if (T < 0) return fail(LISA_ERR_INVALID_ARG, "T=%d < 0", T);
  if (T == 0 || L->B == 0) return ok();
  if (T > L->L_max) return fail(LISA_ERR_INVALID_ARG, "T=%d > L_max=%d", T, L->L_max);
  if (L->dtype != LISA_BF16) return fail(LISA_ERR_UNSUPPORTED, "lisa_indexer_kl supports bf16 storage only");
  if ((s = check_caches(L))) return s;
  if ((s = check_ptr(q, "q")) || (s = check_ptr(qidx, "qidx")) || (s = check_ptr(w, "w")) ||
      (s = check_ptr(kl_out, "kl_out")))
    return s;
  lisa::RowsParams r;
  fill_rows(r, L, T);
  r.q = q; r.qidx = qidx; r.w = w;
  cudaError_t e = lisa::launch_indexer_kl(r, kl_out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "indexer_kl");
  return ok();
}

lisa_status lisa_indexer_topk_noalloc(const lisa_layer *L, const void *qidx, const float *w, int T, int *idx_out,
                                      void *stream) {
  lisa_status s;
  if ((s = check_layer(L))) return s;
  if (T < 0) return fail(LISA_ERR_INVALID_ARG, "T=%d < 0", T);
  if (T == 0 || L->B == 0) return ok();
  if (T > L->L_max) return fail(LISA_ERR_INVALID_ARG, "T=%d > L_max=%d", T, L->L_max);
  if ((s = check_caches(L))) return s;
  if ((s = check_ptr(qidx, "qidx")) || (s = check_ptr(w, "w")) || (s = check_ptr(idx_out, "idx_out"))) return s;
  // one order key per (sequence, KV head, cached position) for every query row of a pass
  const size_t per_row = (size_t)L->B * L->Hkv * round4(L->L_max) * 4;
  if (per_row > (size_t)LISA_NOALLOC_SCRATCH_BYTES)
    return fail(LISA_ERR_UNSUPPORTED,
                "B*Hkv*L_max needs %zu bytes of scratch per query row; the fixed scratch holds %u bytes",
                per_row, (unsigned)LISA_NOALLOC_SCRATCH_BYTES);
  size_t rows = (size_t)LISA_NOALLOC_SCRATCH_BYTES / per_row;
  if (rows > (size_t)kRowChunk) rows = kRowChunk;
  if (rows > (size_t)T) rows = T;
  void *scratch = nullptr;
  if ((s = noalloc_scratch(&scratch))) return s;
  lisa::RowsParams r;
  fill_rows(r, L, T);
  r.qidx = qidx; r.w = w; r.idx = idx_out;
  r.keys = static_cast<uint32_t *>(scratch);   // every slot read is written earlier in the same call
  r.row_chunk = (int)rows;
  r.L_keys = round4(L->L_max);
  set_select_smem(r, L->L_max);
  cudaError_t e = lisa::launch_rows_topk(r, L->dtype, (cudaStream_t)stream, L->L_max);
  if (e != cudaSuccess) return cuda_fail(e, "indexer_topk_noalloc");
  return ok();
}

size_t lisa_workspace_bytes_variant(const lisa_layer *layer, int variant, int T, int op) {
  VariantGeom vg;
  if (check_layer(layer) != LISA_OK || T < 0 || check_variant(layer, variant, vg) != LISA_OK) return 0;
  if (op == LISA_OP_DECODE)
    return vg.row_indexer() ? var_plan(layer, vg, 1, op).total : vg.lin_kv ? 0 : decode_workspace_bytes(layer);
  if (variant == 0 && (op == LISA_OP_PREFILL || op == LISA_OP_INDEXER_TOPK))
    return lisa_workspace_bytes(layer, T, op);            // the default calls (variant 0 runs them)
  if (op == LISA_OP_PREFILL || op == LISA_OP_INDEXER_TOPK) return T ? var_plan(layer, vg, T, op).total : 0;
  return 0;
}

lisa_status lisa_append_cache_variant(const lisa_layer *L, int variant, const void *k, const void *v,
                                      const void *kidx, int T, void *stream) {
  lisa_status s;
  VariantGeom vg;
  if ((s = check_layer(L)) || (s = check_variant(L, variant, vg))) return s;
  if (T < 0) return fail(LISA_ERR_INVALID_ARG, "T=%d < 0", T);
  if (T == 0 || L->B == 0) return ok();
  if (T > L->L_max) return fail(LISA_ERR_INVALID_ARG, "T=%d > L_max=%d", T, L->L_max);
  if ((s = check_caches(L))) return s;
  if ((s = check_ptr(k, "k")) || (s = check_ptr(v, "v")) || (s = check_ptr(kidx, "kidx"))) return s;
  lisa::RowsParams r;
  fill_rows(r, L, T);
  r.k = k; r.v = v;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = lisa::launch_append(r, L->dtype, st);
  if (e == cudaSuccess) e = append_kidx_planes(L, vg, T, kidx, 0, st);
  if (e != cudaSuccess) return cuda_fail(e, "append_cache_variant");
  return ok();
}

lisa_status lisa_indexer_topk_variant(const lisa_layer *L, int variant, const void *qidx, const float *w, int T,
                                      int *idx_out, void *workspace, size_t ws_bytes, void *stream) {
  lisa_status s;
  VariantGeom vg;
  if ((s = check_layer(L)) || (s = check_variant(L, variant, vg))) return s;
  if (variant == 0) return lisa_indexer_topk(L, qidx, w, T, idx_out, workspace, ws_bytes, stream);
  if (T < 0) return fail(LISA_ERR_INVALID_ARG, "T=%d < 0", T);
  if (T == 0 || L->B == 0) return ok();
  if (T > L->L_max) return fail(LISA_ERR_INVALID_ARG, "T=%d > L_max=%d", T, L->L_max);
  if ((s = check_caches(L))) return s;
  if ((s = check_ptr(qidx, "qidx")) || (s = check_ptr(w, "w")) || (s = check_ptr(idx_out, "idx_out"))) return s;
  const VarPlan plan = var_plan(L, vg, T, LISA_OP_INDEXER_TOPK);
  if (!workspace || ws_bytes < plan.total)
    return fail(LISA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace ? ws_bytes : 0, plan.total);
  if ((s = check_ptr(workspace, "workspace"))) return s;
  lisa::RowsParams sel, ph;
  variant_indexer_params(L, vg, T, plan, static_cast<char *>(workspace), qidx, w, idx_out, L->L_max, sel, ph);
  cudaError_t e = lisa::launch_rows_topk(sel, L->dtype, (cudaStream_t)stream, L->L_max, ph.keys ? &ph : nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "indexer_topk_variant");
  return ok();
}

lisa_status lisa_decode_step_variant(const lisa_layer *L, int variant, const void *q, const void *k, const void *v,
                                     const void *kidx, const void *qidx, const float *w, const float *gate_logit,
                                     const void *k_lin, const void *v_lin, int fuse_append, void *out, int *idx_out,
                                     void *workspace, size_t ws_bytes, void *stream) {
  lisa_status s;
  VariantGeom vg;
  if ((s = check_layer(L)) || (s = check_variant(L, variant, vg))) return s;
  if (L->B == 0) return ok();
  if ((s = check_caches(L))) return s;
  if ((s = check_ptr(L->state, "state"))) return s;
  if ((s = check_ptr(q, "q")) || (s = check_ptr(k, "k")) || (s = check_ptr(v, "v")) || (s = check_ptr(kidx, "kidx")) ||
      (s = check_ptr(qidx, "qidx")) || (s = check_ptr(w, "w")) || (s = check_ptr(gate_logit, "gate_logit")) ||
      (s = check_ptr(out, "out")) || (s = check_ptr(idx_out, "idx_out", false)) ||
      (s = check_ptr(k_lin, "k_lin", vg.lin_kv)) || (s = check_ptr(v_lin, "v_lin", vg.lin_kv)))
    return s;
  const int esz = L->dtype == LISA_BF16 ? 2 : 4;
  if (lisa::decode_smem_bytes(L->L_max, L->M, L->Hq / L->Hkv, L->d, L->dI, esz, 8, vg.lin_kv) > kMaxSmem)
    return fail(LISA_ERR_UNSUPPORTED, "L_max=%d needs more shared memory per CTA than a B200 SM has", L->L_max);
  VarPlan plan;
  memset(&plan, 0, sizeof(plan));
  if (vg.row_indexer()) {
    plan = var_plan(L, vg, 1, LISA_OP_DECODE);
    if (!workspace || ws_bytes < plan.total)
      return fail(LISA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace ? ws_bytes : 0, plan.total);
    if ((s = check_ptr(workspace, "workspace"))) return s;
  }
  cudaStream_t st = (cudaStream_t)stream;
  lisa::DecodeParams p;
  memset(&p, 0, sizeof(p));
  p.B = L->B; p.Hq = L->Hq; p.Hkv = L->Hkv; p.G = L->Hq / L->Hkv; p.HI = L->HI; p.R = L->HI / L->Hkv;
  p.D = L->d; p.DI = L->dI; p.M = L->M; p.L_max = L->L_max; p.fuse_append = fuse_append ? 1 : 0;
  p.split_req = L->decode_split;
  p.independent = L->independent ? 1 : 0;
  p.debug_flags = L->debug_flags;
  p.scale = (float)(1.0 / sqrt((double)L->d));
  p.k_cache = L->k_cache; p.v_cache = L->v_cache; p.kidx_cache = L->kidx_cache;
  p.state = L->state; p.pos = L->pos; p.err_word = L->err_word;
  p.q = q; p.k = k; p.v = v; p.kidx = kidx; p.qidx = qidx; p.w = w; p.gate = gate_logit;
  p.out = out; p.idx_out = idx_out;
  if (vg.lin_kv) {
    p.k_lin = k_lin;
    p.v_lin = v_lin;
  }
  // with the row-path indexer the attention kernel reads the lists that the
  // launch before it writes: it always waits for that launch
  if (vg.row_indexer()) p.independent = 0;
  cudaError_t e = cudaSuccess;
  if (vg.row_indexer()) {
    // the new token's indexer keys go into the cache first: the row path reads rows 0..t there
    char *ws = static_cast<char *>(workspace);
    int *idx = idx_out ? idx_out : reinterpret_cast<int *>(ws + plan.idx);
    if (fuse_append) e = append_kidx_planes(L, vg, 1, kidx, 0, st);
    if (e != cudaSuccess) return cuda_fail(e, "decode_step_variant append");
    lisa::RowsParams sel, ph;
    variant_indexer_params(L, vg, 1, plan, ws, qidx, w, idx, L->L_max, sel, ph);
    e = lisa::launch_rows_topk(sel, L->dtype, st, L->L_max, ph.keys ? &ph : nullptr);
    if (e != cudaSuccess) return cuda_fail(e, "decode_step_variant indexer");
    p.sel_ext = idx;
    p.sel_groups = vg.Gs;
    p.kidx = nullptr; p.qidx = nullptr; p.w = nullptr;
    p.idx_out = nullptr;
  } else if (!vg.lin_kv) {
    // the default reading: the same forms as lisa_decode_step
    lisa_status s2;
    if ((s2 = plan_decode_form(L, workspace, ws_bytes, p))) return s2;
  }
  e = lisa::launch_decode(p, L->dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "decode_step_variant");
  return ok();
}

lisa_status lisa_prefill_variant(const lisa_layer *L, int variant, int T, const void *q, const void *k, const void *v,
                                 const void *kidx, const void *qidx, const float *w, const float *gate_logit,
                                 const void *k_lin, const void *v_lin, void *out, int *idx_out, void *workspace,
                                 size_t ws_bytes, void *stream) {
  lisa_status s;
  VariantGeom vg;
  if ((s = check_layer(L)) || (s = check_variant(L, variant, vg))) return s;
  if (variant == 0)
    return lisa_prefill(L, T, q, k, v, kidx, qidx, w, gate_logit, out, idx_out, workspace, ws_bytes, stream);
  if (T < 0) return fail(LISA_ERR_INVALID_ARG, "T=%d < 0", T);
  if (T == 0 || L->B == 0) return ok();
  if (T > L->L_max) return fail(LISA_ERR_INVALID_ARG, "T=%d > L_max=%d", T, L->L_max);
  if ((s = check_caches(L))) return s;
  if ((s = check_ptr(L->state, "state"))) return s;
  if ((s = check_ptr(q, "q")) || (s = check_ptr(k, "k")) || (s = check_ptr(v, "v")) || (s = check_ptr(kidx, "kidx")) ||
      (s = check_ptr(qidx, "qidx")) || (s = check_ptr(w, "w")) || (s = check_ptr(gate_logit, "gate_logit")) ||
      (s = check_ptr(out, "out")) || (s = check_ptr(idx_out, "idx_out", false)) ||
      (s = check_ptr(k_lin, "k_lin", vg.lin_kv)) || (s = check_ptr(v_lin, "v_lin", vg.lin_kv)))
    return s;
  const VarPlan plan = var_plan(L, vg, T, LISA_OP_PREFILL);
  if (!workspace || ws_bytes < plan.total)
    return fail(LISA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace ? ws_bytes : 0, plan.total);
  if ((s = check_ptr(workspace, "workspace"))) return s;
  char *ws = static_cast<char *>(workspace);
  cudaStream_t st = (cudaStream_t)stream;
  int *idx = idx_out ? idx_out : reinterpret_cast<int *>(ws + plan.idx);

  // k, v and the indexer keys (P planes) into the caches
  lisa::RowsParams r;
  fill_rows(r, L, T);
  r.require_pos0 = 1;
  r.k = k; r.v = v;
  cudaError_t e = lisa::launch_append(r, L->dtype, st);
  if (e == cudaSuccess) e = append_kidx_planes(L, vg, T, kidx, 1, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill_variant append");
  // linear branch: with keys / values per query head it runs as Hq groups of one head
  r.q = q; r.gate = gate_logit; r.out = out;
  r.olin = reinterpret_cast<float *>(ws + plan.olin);
  r.dS = reinterpret_cast<float *>(ws + plan.dS);
  r.Ptot = reinterpret_cast<float *>(ws + plan.Ptot);
  {
    lisa::RowsParams rl = r;
    if (vg.lin_kv) {
      rl.Hkv = L->Hq; rl.G = 1;
      rl.k = k_lin; rl.v = v_lin;
    }
    e = lisa::launch_prefill_linear(rl, L->dtype, st);
    if (e != cudaSuccess) return cuda_fail(e, "prefill_variant linear");
  }
  // indexer + top-M in the Gs selection groups
  lisa::RowsParams sel, ph;
  variant_indexer_params(L, vg, T, plan, ws, qidx, w, idx, T, sel, ph);
  sel.require_pos0 = 1;
  ph.require_pos0 = 1;
  e = lisa::launch_rows_topk(sel, L->dtype, st, T, ph.keys ? &ph : nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "prefill_variant indexer");
  // sparse attention + gate: every KV head reads its group's list
  r.idx = idx;
  r.sel_heads = vg.Gs;
  e = lisa::launch_prefill_attend(r, L->dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill_variant attend");
  return ok();
}

lisa_status lisa_project_in(const lisa_layer *L, int variant, const lisa_proj *proj, int T, const void *x, void *q,
                            void *k, void *v, void *qidx, void *kidx, float *w, float *gate_logit, void *stream) {
  lisa_status s;
  VariantGeom vg;
  if ((s = check_layer(L)) || (s = check_variant(L, variant, vg))) return s;
  if (!proj) return fail(LISA_ERR_INVALID_ARG, "proj is NULL");
  if (T < 0) return fail(LISA_ERR_INVALID_ARG, "T=%d < 0", T);
  if (T == 0 || L->B == 0) return ok();
  if (L->dtype != LISA_BF16) return fail(LISA_ERR_UNSUPPORTED, "projections support bf16 storage only");
  if (proj->Hm < 8 || proj->Hm % 8) return fail(LISA_ERR_UNSUPPORTED, "Hm=%d is not a positive multiple of 8", proj->Hm);
  if ((s = check_ptr(proj->W_in, "W_in")) || (s = check_ptr(x, "x")) || (s = check_ptr(q, "q")) ||
      (s = check_ptr(k, "k")) || (s = check_ptr(v, "v")) || (s = check_ptr(qidx, "qidx")) ||
      (s = check_ptr(kidx, "kidx")) || (s = check_ptr(w, "w")) || (s = check_ptr(gate_logit, "gate_logit")))
    return s;
  lisa::ProjParams p;
  memset(&p, 0, sizeof(p));
  p.rows = L->B * T;
  p.K = proj->Hm;
  p.err_word = L->err_word;
  const int widths[7] = {L->Hq * L->d, L->Hkv * L->d, L->Hkv * L->d, L->HI * L->dI, vg.P * L->dI, L->HI, L->Hq};
  void *ptrs[7] = {q, k, v, qidx, kidx, w, gate_logit};
  int c = 0;
  for (int i = 0; i < 7; ++i) {
    p.seg[i].c0 = c;
    p.seg[i].width = widths[i];
    p.seg[i].ptr = ptrs[i];
    p.seg[i].f32 = i >= 5;
    c += widths[i];
  }
  p.nseg = 7;
  p.N = c;
  cudaError_t e = lisa::launch_proj(p, x, proj->W_in, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "project_in");
  return ok();
}

lisa_status lisa_project_out(const lisa_layer *L, const lisa_proj *proj, int T, const void *o, void *y, void *stream) {
  lisa_status s;
  if ((s = check_layer(L))) return s;
  if (!proj) return fail(LISA_ERR_INVALID_ARG, "proj is NULL");
  if (T < 0) return fail(LISA_ERR_INVALID_ARG, "T=%d < 0", T);
  if (T == 0 || L->B == 0) return ok();
  if (L->dtype != LISA_BF16) return fail(LISA_ERR_UNSUPPORTED, "projections support bf16 storage only");
  if (proj->Hm < 8 || proj->Hm % 8) return fail(LISA_ERR_UNSUPPORTED, "Hm=%d is not a positive multiple of 8", proj->Hm);
  if ((s = check_ptr(proj->W_o, "W_o")) || (s = check_ptr(o, "o")) || (s = check_ptr(y, "y"))) return s;
  lisa::ProjParams p;
  memset(&p, 0, sizeof(p));
  p.rows = L->B * T;
  p.K = L->Hq * L->d;
  p.N = proj->Hm;
  p.err_word = L->err_word;
  p.nseg = 1;
  p.seg[0].c0 = 0;
  p.seg[0].width = proj->Hm;
  p.seg[0].ptr = y;
  p.seg[0].f32 = 0;
  cudaError_t e = lisa::launch_proj(p, o, proj->W_o, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "project_out");
  return ok();
}

}  // extern "C"
