// api.cpp -- the C ABI of libmad (include/mad.h): argument validation,
// context lifetime, double-buffer bookkeeping and dispatch to the kernels.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法: analyse the terms and preallocate the CSR from
// topology (mad_create), run the patch-parallel evaluate / differentiate /
// assemble kernel (mad_eval), the matrix-free product (mad_hvp), and insert
// runtime pairs into a double-buffered CSR on the GPU (mad_add_pairs).  After
// mad_create nothing here allocates or synchronises (except the documented
// host-buffer and status entry points).
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "mad_internal.h"

using namespace mad;

struct mad_ctx {
  int V = 0, nF = 0, E = 0, dof = 0, dtype = 0, esz = 4;
  int nnzb_base = 0, capacity = 0, max_pairs = 0;
  mad_opts opts{};
  int device = 0;
  PatternDev pat{};
  int32_t* F_dev = nullptr;
  int32_t* base_nnzb_dev = nullptr;
  // patches
  int n_patches = 0, nv_max = 0, no_max = 0, slots_max = 0;
  int grid_base = 0, grid_pairs = 0;  // persistent grids (no pairs / pairs)
  // staging capacity in dtype elements: the largest patch's mesh-pattern rows
  // plus 16-byte alignment room per run; stage_cap adds a reserve for pair
  // blocks
  int stage_base = 0;
  int stage_cap = 0;
  PatchHdr* hdr = nullptr;
  int32_t* vgid = nullptr;
  uint2* meta = nullptr;
  uint32_t* runs = nullptr;
  EdgeLut* elut = nullptr;
  int32_t* eid = nullptr;
  int32_t* ecol = nullptr;
  FaceLut* flut = nullptr;
  int32_t* fcol = nullptr;
  uint16_t* slot_lidx = nullptr;
  int32_t* slot_eid = nullptr;
  int rho = 0;  // staging room per row for pair blocks (pairs active)
  // row-streaming kernel tables
  int rows_s0 = 0;
  int2* rows_slots = nullptr;
  uint32_t* rows_meta = nullptr;
  int32_t* rows_ofl_ptr = nullptr;
  int2* rows_ofl = nullptr;
  std::vector<int32_t> rp_host;    // the mesh pattern's row_ptr (host copy)
  int4* rows_ctile = nullptr;      // compact slots (nullptr when they do not fit)
  uint32_t* rows_cslots = nullptr;
  // face rows of the same kernel (rows_sf == 0: face terms use the patch kernel)
  int rows_sf = 0;
  int4* rows_fslots = nullptr;
  int32_t* rows_fofl_ptr = nullptr;
  int4* rows_fofl = nullptr;
  int32_t* rows_fcslots = nullptr;
  int32_t* rows_fcofl = nullptr;
  void* face_hv = nullptr;  // [nF][3][2] scratch of the face Hessian-vector product
  void* pe_xr = nullptr;    // [2*max_pairs][4] partner position + rest per pair entry
  double* epart = nullptr;
  size_t smem_eval = 0, smem_hvp = 0;
  // dynamic pattern
  DynBuf buf[2];
  int active = -1;  // -1: mesh pattern, no pairs
  VfSet vfs;        // the installed vertex-face term set (mad_add_vf)
  // insertion scratch
  int32_t *cnt = nullptr, *tsum = nullptr, *newcnt = nullptr, *pe_pid = nullptr,
          *status = nullptr;
  // mad_eval_host staging (allocated on first use)
  void *hx = nullptr, *hg = nullptr, *hH = nullptr;
  double* he = nullptr;
  int64_t device_bytes = 0;
  std::vector<void*> allocs;
  std::string err;
};

namespace {

constexpr int kMaxPatchOwned = 256;  // threads per block of the patch kernels
std::string g_create_error;

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

template <typename P>
cudaError_t dev_alloc(mad_ctx* c, P** p, size_t bytes) {
  if (bytes == 0) bytes = 16;
  void* q = nullptr;
  cudaError_t e = cudaMalloc(&q, bytes);
  if (e != cudaSuccess) return e;
  c->allocs.push_back(q);
  c->device_bytes += (int64_t)bytes;
  *p = reinterpret_cast<P*>(q);
  return cudaSuccess;
}

template <typename P>
cudaError_t upload(mad_ctx* c, P** p, const std::vector<P>& v) {
  cudaError_t e = dev_alloc(c, p, sizeof(P) * v.size());
  if (e != cudaSuccess || v.empty()) return e;
  return cudaMemcpy(*p, v.data(), sizeof(P) * v.size(), cudaMemcpyHostToDevice);
}

void free_ctx(mad_ctx* c) {
  if (!c) return;
  cudaDeviceSynchronize();
  for (void* p : c->allocs) cudaFree(p);
  cudaFree(c->pat.rp);
  cudaFree(c->pat.ci);
  cudaFree(c->pat.diag);
  cudaFree(c->pat.edges);
  cudaFree(c->hx);
  cudaFree(c->hg);
  cudaFree(c->hH);
  cudaFree(c->he);
  delete c;
}

mad_status fail(mad_ctx* c, mad_status st, const std::string& msg) {
  if (c) c->err = msg;
  return st;
}

mad_status cuda_fail(mad_ctx* c, cudaError_t e, const char* where) {
  return fail(c, MAD_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

EvalLaunch eval_launch(const mad_ctx* c) {
  EvalLaunch L;
  L.dtype = c->dtype;
  L.dof = c->dof;
  L.n_patches = c->n_patches;
  L.nv_max = c->nv_max;
  L.no_max = c->no_max;
  L.slots_max = c->slots_max;
  L.grid = c->active < 0 ? c->grid_base : c->grid_pairs;
  // without pair blocks the rows never outgrow the mesh pattern, so the
  // kernel is launched with less shared memory (more blocks per SM)
  L.stage_cap = c->active < 0 ? std::min(c->stage_base, c->stage_cap) : c->stage_cap;
  L.hdr = c->hdr;
  L.vgid = c->vgid;
  L.meta = c->meta;
  L.elut = c->elut;
  L.eid = c->eid;
  L.ecol = c->ecol;
  L.flut = c->flut;
  L.fcol = c->fcol;
  L.slot_lidx = c->slot_lidx;
  L.slot_eid = c->slot_eid;
  L.runs = c->runs;
  L.rho = c->active < 0 ? 0 : c->rho;
  L.epart = c->epart;
  if (c->active < 0) {
    L.rp = c->pat.rp;
    L.prow = nullptr;
    L.pe_col = nullptr;
    L.pe_pos = nullptr;
    L.pe_rest = nullptr;
  } else {
    const DynBuf& b = c->buf[c->active];
    L.rp = b.rp;
    L.prow = b.prow;  // the pair layout applies even when pair terms are off
    L.pe_col = b.pe_col;
    L.pe_pos = b.pe_pos;
    L.pe_rest = b.pe_rest;
  }
  return L;
}

RowsLaunch rows_launch(const mad_ctx* c) {
  RowsLaunch L;
  L.dtype = c->dtype;
  L.dof = c->dof;
  L.V = c->V;
  L.s0 = c->rows_s0;
  L.rho = c->active < 0 ? 0 : c->rho;
  L.slots = c->rows_slots;
  L.meta = c->rows_meta;
  L.ofl_ptr = c->rows_ofl_ptr;
  L.ofl = c->rows_ofl;
  L.ctile = c->rows_ctile;
  L.cslots = c->rows_cslots;
  L.sf = c->rows_sf;
  L.fslots = c->rows_fslots;
  L.fofl_ptr = c->rows_fofl_ptr;
  L.fofl = c->rows_fofl;
  L.fcslots = c->rows_fcslots;
  L.fcofl = c->rows_fcofl;
  L.nF = c->nF;
  L.F = c->F_dev;
  L.fhv = c->face_hv;
  L.epart = c->epart;
  if (c->active < 0) {
    L.rp = c->pat.rp;
    L.prow = nullptr;
    L.pe_col = nullptr;
    L.pe_pos = nullptr;
    L.pe_rest = nullptr;
    L.pmask = nullptr;
  } else {
    const DynBuf& b = c->buf[c->active];
    L.rp = b.rp;
    L.prow = b.prow;
    L.pe_col = b.pe_col;
    L.pe_pos = b.pe_pos;
    L.pe_rest = b.pe_rest;
    L.pmask = b.pmask;
    L.pe_xr = c->pe_xr;
  }
  return L;
}

// The vertex-face pass reads the active pattern: the mesh pattern, or the
// buffer that the last mad_add_pairs filled.
VfLaunch vf_launch(const mad_ctx* c, const mad_terms* t, const void* x) {
  VfLaunch L;
  L.n = t->vf_n;
  L.V = c->V;
  L.nF = c->nF;
  L.vf = t->vf;
  L.rest = t->vf_rest;
  L.k = t->vf_k;
  L.F = c->F_dev;
  L.x = x;
  L.rp = c->active < 0 ? c->pat.rp : c->buf[c->active].rp;
  L.ci = c->active < 0 ? c->pat.ci : c->buf[c->active].ci;
  L.status = c->status;
  L.generic = (t->flags & MAD_EVAL_GENERIC_AD) != 0;
  return L;
}

// Every term set goes to the row-streaming kernel unless the caller asks for
// the patch kernel or the scatter mode, or face terms meet a mesh whose face
// rows could not be built.
bool use_rows(const mad_ctx* c, const mad_terms* t) {
  if (t->flags & (MAD_EVAL_EDGE_SCATTER | MAD_EVAL_PATCH_STAGED)) return false;
  return !(t->mask & (MAD_TERM_SYMDIR | MAD_TERM_AREA | MAD_TERM_ARAP)) || c->nF == 0 ||
         c->rows_sf > 0;
}

mad_status check_terms(mad_ctx* c, const mad_terms* t) {
  if (!t) return fail(c, MAD_ERR_INVALID_ARG, "terms is NULL");
  const uint32_t known = MAD_TERM_SPRING | MAD_TERM_INERTIA | MAD_TERM_SYMDIR | MAD_TERM_PAIR |
                         MAD_TERM_AREA | MAD_TERM_ARAP | MAD_TERM_VF;
  if (t->mask & ~known) return fail(c, MAD_ERR_INVALID_ARG, "unknown term bits in mask");
  if (t->mask & MAD_TERM_VF) {
    if (c->dof != 3) return fail(c, MAD_ERR_UNIMPLEMENTED, "vertex-face terms need dof 3");
    if (t->mask & MAD_TERM_PAIR)
      return fail(c, MAD_ERR_UNIMPLEMENTED, "vertex-face terms with pair terms in one mask");
    if (t->vf_n < 0) return fail(c, MAD_ERR_INVALID_ARG, "vf_n < 0");
    if (t->vf_n > 0 && !t->vf_rest)
      return fail(c, MAD_ERR_INVALID_ARG, "vertex-face terms need vf_rest");
    if (t->vf_n > 0 && !t->vf && t->vf_n != c->vfs.n)
      return fail(c, MAD_ERR_INVALID_ARG,
                  "vf is NULL but vf_n is not the size of the set installed by mad_add_vf");
  }
  if (t->flags & ~(uint32_t)(MAD_EVAL_FULL_STENCIL_AD | MAD_EVAL_EDGE_SCATTER |
                             MAD_EVAL_PATCH_STAGED | MAD_EVAL_GENERIC_AD))
    return fail(c, MAD_ERR_INVALID_ARG, "unknown evaluation flags");
  if ((t->flags & MAD_EVAL_GENERIC_AD) && (t->flags & MAD_EVAL_FULL_STENCIL_AD))
    return fail(c, MAD_ERR_INVALID_ARG, "MAD_EVAL_GENERIC_AD with MAD_EVAL_FULL_STENCIL_AD");
  if ((t->flags & MAD_EVAL_GENERIC_AD) &&
      (t->flags & (MAD_EVAL_EDGE_SCATTER | MAD_EVAL_PATCH_STAGED)))
    return fail(c, MAD_ERR_UNIMPLEMENTED, "MAD_EVAL_GENERIC_AD runs on the row kernel only");
  if ((t->mask & MAD_TERM_SPRING) && c->E > 0 && !t->spring_rest)
    return fail(c, MAD_ERR_INVALID_ARG, "spring term active but spring_rest is NULL");
  if ((t->mask & MAD_TERM_INERTIA) && c->V > 0 && !t->inertia_xt)
    return fail(c, MAD_ERR_INVALID_ARG, "inertia term active but inertia_xt is NULL");
  if (t->mask & MAD_TERM_SYMDIR) {
    if (c->dof != 2)
      return fail(c, MAD_ERR_UNIMPLEMENTED, "symmetric Dirichlet term needs dof 2");
    if (c->nF > 0 && (!t->face_Minv || !t->face_area))
      return fail(c, MAD_ERR_INVALID_ARG, "symmetric Dirichlet term needs face_Minv and face_area");
  }
  if (t->mask & MAD_TERM_ARAP) {
    if (c->dof != 2) return fail(c, MAD_ERR_UNIMPLEMENTED, "ARAP term needs dof 2");
    if (c->nF > 0 && (!t->face_Minv || !t->face_area))
      return fail(c, MAD_ERR_INVALID_ARG, "ARAP term needs face_Minv and face_area");
    // only the row-streaming kernel evaluates it
    if (t->flags & (MAD_EVAL_EDGE_SCATTER | MAD_EVAL_PATCH_STAGED))
      return fail(c, MAD_ERR_UNIMPLEMENTED, "ARAP term needs the row kernel");
    if (c->nF > 0 && c->rows_sf == 0)
      return fail(c, MAD_ERR_UNIMPLEMENTED, "ARAP term: a mesh row too long for the face rows");
  }
  if (t->mask & MAD_TERM_AREA) {
    if (c->dof != 3)
      return fail(c, MAD_ERR_UNIMPLEMENTED, "area-preservation term needs dof 3");
    if (c->nF > 0 && !t->face_area)
      return fail(c, MAD_ERR_INVALID_ARG, "area-preservation term needs face_area");
    // only the row-streaming kernel evaluates it
    if (t->flags & (MAD_EVAL_EDGE_SCATTER | MAD_EVAL_PATCH_STAGED))
      return fail(c, MAD_ERR_UNIMPLEMENTED, "area-preservation term needs the row kernel");
    if (c->nF > 0 && c->rows_sf == 0)
      return fail(c, MAD_ERR_UNIMPLEMENTED,
                  "area-preservation term: a mesh row too long for the face rows");
  }
  return MAD_OK;
}

}  // namespace

extern "C" {

void mad_default_opts(mad_opts* o) {
  if (!o) return;
  std::memset(o, 0, sizeof(*o));
  o->patch_faces = 512;
  o->slack = 0.10f;
  o->max_pairs = 0;
  o->part_xyz = nullptr;
  o->part_dim = 0;
  o->smem_budget = 0;
}

mad_status mad_create(int32_t V, int32_t nF, const int32_t* F, int32_t dof, mad_dtype dt,
                      const mad_opts* o, void* stream, mad_ctx** out) {
  g_create_error.clear();
  if (!out) {
    g_create_error = "out is NULL";
    return MAD_ERR_INVALID_ARG;
  }
  *out = nullptr;
  if (V < 0 || nF < 0 || (nF > 0 && !F) || (dof != 2 && dof != 3) ||
      (dt != MAD_F32 && dt != MAD_F64)) {
    g_create_error = "invalid V, nF, F, dof or dtype";
    return MAD_ERR_INVALID_ARG;
  }
  for (int64_t f = 0; f < nF; ++f) {
    const int32_t a = F[3 * f], b = F[3 * f + 1], cc = F[3 * f + 2];
    if (a < 0 || a >= V || b < 0 || b >= V || cc < 0 || cc >= V || a == b || b == cc ||
        a == cc) {
      char buf[128];
      std::snprintf(buf, sizeof buf, "face %lld has an index out of range or repeated",
                    (long long)f);
      g_create_error = buf;
      return MAD_ERR_INVALID_ARG;
    }
  }
  mad_opts opts;
  mad_default_opts(&opts);
  if (o) {
    if (o->patch_faces > 0) opts.patch_faces = o->patch_faces;
    if (o->slack >= 0.f) opts.slack = o->slack;
    opts.max_pairs = o->max_pairs;
    opts.part_xyz = o->part_xyz;
    opts.part_dim = o->part_dim;
    opts.smem_budget = o->smem_budget;
    if (opts.part_xyz && opts.part_dim != 2 && opts.part_dim != 3) {
      g_create_error = "part_dim must be 2 or 3";
      return MAD_ERR_INVALID_ARG;
    }
  }
  mad_ctx* c = new mad_ctx();
  c->V = V;
  c->nF = nF;
  c->dof = dof;
  c->dtype = dt;
  c->esz = dt == MAD_F64 ? 8 : 4;
  c->opts = opts;
  cudaGetDevice(&c->device);
  cudaStream_t s = as_stream(stream);
  cudaError_t e;
  std::string msg;
  const int B = dof * dof;
  int smem_optin = 0;

#define CREATE_CK(x)                                                  \
  do {                                                                \
    e = (x);                                                          \
    if (e != cudaSuccess) {                                           \
      g_create_error = std::string(#x) + ": " + cudaGetErrorString(e); \
      free_ctx(c);                                                    \
      return e == cudaErrorMemoryAllocation ? MAD_ERR_OOM : MAD_ERR_CUDA; \
    }                                                                 \
  } while (0)

  // 1. topology on the GPU: pattern + edges
  CREATE_CK(dev_alloc(c, &c->F_dev, sizeof(int32_t) * 3 * (size_t)nF));
  if (nF > 0)
    CREATE_CK(cudaMemcpyAsync(c->F_dev, F, sizeof(int32_t) * 3 * (size_t)nF,
                              cudaMemcpyHostToDevice, s));
  msg = build_pattern_gpu(V, nF, c->F_dev, s, c->pat);
  if (!msg.empty()) {
    g_create_error = "pattern: " + msg;
    free_ctx(c);
    return MAD_ERR_CUDA;
  }
  c->nnzb_base = c->pat.nnzb;
  c->E = c->pat.E;
  CREATE_CK(dev_alloc(c, &c->base_nnzb_dev, sizeof(int32_t)));
  CREATE_CK(cudaMemcpy(c->base_nnzb_dev, &c->nnzb_base, sizeof(int32_t), cudaMemcpyHostToDevice));

  // 2. patches on the host
  {
    std::vector<int32_t> rp(V + 1), ci(c->nnzb_base);
    CREATE_CK(cudaMemcpy(rp.data(), c->pat.rp, sizeof(int32_t) * (V + 1), cudaMemcpyDeviceToHost));
    if (c->nnzb_base > 0)
      CREATE_CK(cudaMemcpy(ci.data(), c->pat.ci, sizeof(int32_t) * c->nnzb_base,
                           cudaMemcpyDeviceToHost));
    const int budget = opts.smem_budget > 0 ? opts.smem_budget : 72 * 1024;
    const int max_stage_blocks = std::max(1, budget / (B * c->esz));
    int target = opts.patch_faces;
    if (nF > 0)
      target = (int)std::max<long long>(1, std::llround((double)opts.patch_faces * V / nF));
    target = std::min(target, kMaxPatchOwned);  // one owned vertex per thread
    HostPatches hp;
    msg = build_patches(V, nF, F, rp.data(), ci.data(), opts.part_xyz, opts.part_dim, target,
                        max_stage_blocks, hp);
    if (!msg.empty()) {
      g_create_error = "patches: " + msg;
      free_ctx(c);
      return MAD_ERR_UNIMPLEMENTED;
    }
    c->n_patches = (int)hp.hdr.size();
    c->nv_max = std::max(1, hp.nv_max);
    c->no_max = std::max(1, hp.no_max);
    c->slots_max = std::max(1, hp.slots_max);
    // staging room: the largest patch's rows plus a reserve for pair blocks
    if (c->no_max > kMaxPatchOwned) {
      g_create_error = "patch with more owned vertices than threads per block";
      free_ctx(c);
      return MAD_ERR_UNIMPLEMENTED;
    }
    // staging: rows at a fixed stride per patch; with pairs active every row
    // gets rho spare blocks (rows that outgrow their run's window are
    // assembled in place in H)
    c->rho = 2;
    size_t st0 = 1, st1 = 1;
    for (const PatchHdr& h : hp.hdr) {
      st0 = std::max(st0, patch_stage_elems(h, dof, c->esz, 0));
      st1 = std::max(st1, patch_stage_elems(h, dof, c->esz, c->rho));
    }
    c->stage_base = (int)st0;
    c->stage_cap = (int)st1;
    CREATE_CK(upload(c, &c->hdr, hp.hdr));
    CREATE_CK(upload(c, &c->vgid, hp.vgid));
    CREATE_CK(upload(c, &c->meta, hp.meta));
    CREATE_CK(upload(c, &c->elut, hp.elut));
    CREATE_CK(upload(c, &c->eid, hp.eid));
    CREATE_CK(upload(c, &c->ecol, hp.ecol));
    CREATE_CK(upload(c, &c->flut, hp.flut));
    CREATE_CK(upload(c, &c->fcol, hp.fcol));
    CREATE_CK(upload(c, &c->slot_lidx, hp.slot_lidx));
    CREATE_CK(upload(c, &c->slot_eid, hp.slot_eid));
    CREATE_CK(upload(c, &c->runs, hp.runs));
    CREATE_CK(dev_alloc(c, &c->epart,
                        sizeof(double) * std::max({1, c->n_patches, rows_blocks(V)})));
    HostRowTables rt;
    msg = build_row_tables(V, rp.data(), ci.data(), 8, rt);
    if (!msg.empty()) {
      g_create_error = "row tables: " + msg;
      free_ctx(c);
      return MAD_ERR_UNIMPLEMENTED;
    }
    c->rows_s0 = rt.s0;
    c->rp_host = rp;
    CREATE_CK(upload(c, &c->rows_slots, rt.slots));
    CREATE_CK(upload(c, &c->rows_meta, rt.meta));
    CREATE_CK(upload(c, &c->rows_ofl_ptr, rt.ofl_ptr));
    CREATE_CK(upload(c, &c->rows_ofl, rt.ofl));
    if (!rt.cslots.empty()) {
      CREATE_CK(upload(c, &c->rows_ctile, rt.ctile));
      CREATE_CK(upload(c, &c->rows_cslots, rt.cslots));
    }
    if (nF > 0) {
      HostFaceRows fr;
      if (build_face_rows(V, nF, F, rp.data(), ci.data(), fr).empty()) {
        c->rows_sf = fr.sf;
        CREATE_CK(upload(c, &c->rows_fslots, fr.slots));
        CREATE_CK(upload(c, &c->rows_fofl_ptr, fr.ofl_ptr));
        CREATE_CK(upload(c, &c->rows_fofl, fr.ofl));
        CREATE_CK(upload(c, &c->rows_fcslots, fr.cslots));
        CREATE_CK(upload(c, &c->rows_fcofl, fr.cofl));
        char* hv = nullptr;
        CREATE_CK(dev_alloc(c, &hv, (size_t)c->esz * 3 * dof * (size_t)nF));
        c->face_hv = hv;
      }
    }
  }
  // 3. shared memory of the patch kernels
  CREATE_CK(cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                   c->device));
  {
    EvalLaunch L = eval_launch(c);
    L.stage_cap = c->stage_cap;
    // the static shared arrays of the kernels take a few hundred bytes
    const size_t limit = (size_t)smem_optin > 1024 ? (size_t)smem_optin - 1024 : 0;
    c->smem_eval = eval_smem_bytes(L, false);
    if (c->smem_eval > limit) {  // drop the pair reserve first
      c->rho = 0;
      c->stage_cap = c->stage_base;
      L.stage_cap = c->stage_cap;
      c->smem_eval = eval_smem_bytes(L, false);
    }
    c->smem_hvp = eval_smem_bytes(L, true);
    if (c->smem_eval > limit || c->smem_hvp > limit) {
      g_create_error = "patch tables exceed the shared memory of one CUDA block";
      free_ctx(c);
      return MAD_ERR_UNIMPLEMENTED;
    }
    CREATE_CK(eval_set_smem_limits(dt, dof, std::max(c->smem_eval, c->smem_hvp)));
    {
      RowsLaunch R = rows_launch(c);
      R.rho = c->rho;
      CREATE_CK(rows_set_smem_limits(dt, dof, rows_smem_bytes(R)));
    }
    L.stage_cap = c->stage_base;
    L.rho = 0;
    c->grid_base = eval_grid(L);
    L.stage_cap = c->stage_cap;
    L.rho = c->rho;
    c->grid_pairs = eval_grid(L);
  }
  // 4. dynamic CSR double buffer and insertion scratch
  {
    const double cap = std::ceil((1.0 + (double)opts.slack) * (double)c->nnzb_base);
    if (cap * B >= 2147483647.0) {
      g_create_error = "capacity * block size exceeds int32 element offsets";
      free_ctx(c);
      return MAD_ERR_UNIMPLEMENTED;
    }
    c->capacity = (int)cap;
    c->max_pairs = opts.max_pairs > 0 ? opts.max_pairs
                                      : std::max(1024, (c->capacity - c->nnzb_base) / 2);
    const size_t pe = 2 * (size_t)c->max_pairs;
    for (int k = 0; k < 2; ++k) {
      DynBuf& b = c->buf[k];
      CREATE_CK(dev_alloc(c, &b.rp, sizeof(int32_t) * (V + 1)));
      CREATE_CK(dev_alloc(c, &b.ci, sizeof(int32_t) * (size_t)c->capacity));
      CREATE_CK(dev_alloc(c, &b.nnzb, sizeof(int32_t)));
      CREATE_CK(dev_alloc(c, &b.prow, sizeof(int32_t) * (V + 1)));
      CREATE_CK(dev_alloc(c, &b.pmask, sizeof(uint32_t) * std::max(1, V)));
      CREATE_CK(dev_alloc(c, &b.pe_col, sizeof(int32_t) * pe));
      CREATE_CK(dev_alloc(c, &b.pe_pos, sizeof(int32_t) * pe));
      char* rest_buf = nullptr;
      CREATE_CK(dev_alloc(c, &rest_buf, (size_t)c->esz * pe));
      b.pe_rest = rest_buf;
    }
    CREATE_CK(dev_alloc(c, &c->pe_xr, (size_t)c->esz * 4 * pe));
    CREATE_CK(dev_alloc(c, &c->cnt, sizeof(int32_t) * (V + 1)));
    CREATE_CK(cudaMemsetAsync(c->cnt, 0, sizeof(int32_t) * (V + 1), s));
    CREATE_CK(dev_alloc(c, &c->tsum, sizeof(int32_t) * pair_scratch_elems(V)));
    CREATE_CK(cudaMemsetAsync(c->tsum, 0, sizeof(int32_t) * pair_scratch_elems(V), s));
    CREATE_CK(dev_alloc(c, &c->newcnt, sizeof(int32_t) * (V + 1)));
    CREATE_CK(dev_alloc(c, &c->pe_pid, sizeof(int32_t) * pe));
    CREATE_CK(dev_alloc(c, &c->status, sizeof(int32_t)));
    CREATE_CK(cudaMemsetAsync(c->status, 0, sizeof(int32_t), s));
    // vertex-face term sets: each term takes three pairs of the pair capacity
    VfSet& vs = c->vfs;
    vs.max_terms = c->max_pairs / 3;
    const size_t mt = (size_t)vs.max_terms;
    CREATE_CK(dev_alloc(c, &vs.terms, sizeof(int32_t) * 2 * std::max<size_t>(mt, 1)));
    CREATE_CK(dev_alloc(c, &vs.pairs, sizeof(int32_t) * 6 * std::max<size_t>(mt, 1)));
    char* zr = nullptr;
    CREATE_CK(dev_alloc(c, &zr, (size_t)c->esz * 3 * std::max<size_t>(mt, 1)));
    CREATE_CK(cudaMemsetAsync(zr, 0, (size_t)c->esz * 3 * std::max<size_t>(mt, 1), s));
    vs.zero_rest = zr;
    CREATE_CK(dev_alloc(c, &vs.vrow, sizeof(int32_t) * (V + 1)));
    CREATE_CK(dev_alloc(c, &vs.ent, sizeof(int32_t) * 32 * std::max<size_t>(mt, 1)));
    CREATE_CK(dev_alloc(c, &vs.scan_tmp, sizeof(int32_t) * scan_tmp_elems(V)));
    CREATE_CK(dev_alloc(c, &vs.epart,
                        sizeof(double) * std::max<size_t>(1, (mt + 255) / 256)));
    CREATE_CK(dev_alloc(c, &vs.vslot, sizeof(int32_t) * 4 * std::max<size_t>(mt, 1)));
    char* rec = nullptr;
    CREATE_CK(dev_alloc(c, &rec, (size_t)c->esz * 160 * std::max<size_t>(mt, 1)));
    vs.rec = rec;
  }
  c->device_bytes += (int64_t)sizeof(int32_t) *
                     ((V + 1) + 2 * (int64_t)c->nnzb_base + V + 2 * (int64_t)c->E);
  CREATE_CK(cudaStreamSynchronize(s));
#undef CREATE_CK
  *out = c;
  return MAD_OK;
}

mad_status mad_info(const mad_ctx* c, mad_info_t* info) {
  if (!c || !info) return MAD_ERR_INVALID_ARG;
  info->V = c->V;
  info->nF = c->nF;
  info->E = c->E;
  info->dof = c->dof;
  info->dtype = c->dtype;
  info->nnzb_base = c->nnzb_base;
  info->capacity_blocks = c->capacity;
  info->max_pairs = c->max_pairs;
  info->n_patches = c->n_patches;
  info->max_patch_vertices = c->nv_max;
  info->max_patch_owned = c->no_max;
  info->smem_bytes = (int32_t)c->smem_eval;
  info->device_bytes = c->device_bytes;
  info->row_slot_bytes = c->rows_cslots ? 4 : 8;
  return MAD_OK;
}

mad_status mad_edges(const mad_ctx* c, const int32_t** ij, int32_t* E) {
  if (!c || !ij || !E) return MAD_ERR_INVALID_ARG;
  *ij = c->pat.edges;
  *E = c->E;
  return MAD_OK;
}

mad_status mad_pattern(const mad_ctx* c, const int32_t** row_ptr, const int32_t** col_idx,
                       const int32_t** nnzb_dev) {
  if (!c || !row_ptr || !col_idx) return MAD_ERR_INVALID_ARG;
  if (c->active < 0) {
    *row_ptr = c->pat.rp;
    *col_idx = c->pat.ci;
    if (nnzb_dev) *nnzb_dev = c->base_nnzb_dev;
  } else {
    *row_ptr = c->buf[c->active].rp;
    *col_idx = c->buf[c->active].ci;
    if (nnzb_dev) *nnzb_dev = c->buf[c->active].nnzb;
  }
  return MAD_OK;
}

mad_status mad_eval(mad_ctx* c, const void* x, const mad_terms* t, void* g, void* H_vals,
                    double* energy, void* stream) {
  if (!c) return MAD_ERR_INVALID_ARG;
  mad_status st = check_terms(c, t);
  if (st != MAD_OK) return st;
  if (c->V > 0 && (!x || !g || !H_vals))
    return fail(c, MAD_ERR_INVALID_ARG, "x, g and H_vals must be device pointers");
  cudaError_t e;
  // installed vertex-face terms without area terms: the term pass first,
  // then the row kernel gathers each row's share into its staged row
  const bool vf_in_rows = (t->mask & MAD_TERM_VF) && t->vf_n > 0 && !t->vf &&
                          !(t->mask & MAD_TERM_AREA) && use_rows(c, t) && c->active >= 0;
  if (use_rows(c, t)) {
    RowsLaunch R = rows_launch(c);
    if (vf_in_rows) {
      e = launch_vf_term_pass(c->dtype, c->vfs, vf_launch(c, t, x), as_stream(stream));
      if (e != cudaSuccess) return cuda_fail(c, e, "mad_eval vertex-face term pass");
      R.vrow = c->vfs.vrow;
      R.vent = c->vfs.ent;
      R.vrec = c->vfs.rec;
    }
    e = launch_rows_eval(R, *t, x, g, H_vals, energy, as_stream(stream));
  } else {
    e = launch_eval(eval_launch(c), *t, x, g, H_vals, energy, as_stream(stream));
  }
  if (e != cudaSuccess) return cuda_fail(c, e, "mad_eval launch");
  if ((t->mask & MAD_TERM_VF) && t->vf_n > 0 && !vf_in_rows) {
    // t->vf given: one thread per term, atomics; else the installed set,
    // gathered per row
    e = t->vf ? launch_vf_eval(c->dtype, vf_launch(c, t, x), g, H_vals, energy, as_stream(stream))
              : launch_vf_rows_eval(c->dtype, c->vfs, vf_launch(c, t, x), g, H_vals, energy,
                                    as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(c, e, "mad_eval vertex-face launch");
  }
  return MAD_OK;
}

mad_status mad_hvp(mad_ctx* c, const void* x, const mad_terms* t, const void* v, void* y,
                   void* stream) {
  if (!c) return MAD_ERR_INVALID_ARG;
  mad_status st = check_terms(c, t);
  if (st != MAD_OK) return st;
  if (c->V > 0 && (!x || !v || !y))
    return fail(c, MAD_ERR_INVALID_ARG, "x, v and y must be device pointers");
  cudaError_t e = use_rows(c, t) ? launch_rows_hvp(rows_launch(c), *t, x, v, y, as_stream(stream))
                              : launch_hvp(eval_launch(c), *t, x, v, y, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(c, e, "mad_hvp launch");
  if ((t->mask & MAD_TERM_VF) && t->vf_n > 0) {
    e = t->vf ? launch_vf_hvp(c->dtype, vf_launch(c, t, x), v, y, as_stream(stream))
              : launch_vf_rows_hvp(c->dtype, c->vfs, vf_launch(c, t, x), v, y, as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(c, e, "mad_hvp vertex-face launch");
  }
  return MAD_OK;
}

mad_status mad_eval_shard(mad_ctx* c, int32_t nranks, const int32_t* row_begin,
                          const void* const* x_parts, int32_t rank, const mad_terms* t,
                          void* g_part, void* H_part, double* energy, void* stream) {
  if (!c) return MAD_ERR_INVALID_ARG;
  mad_status st = check_terms(c, t);
  if (st != MAD_OK) return st;
  if (nranks < 1 || nranks > MAD_MAX_SHARDS || !row_begin || !x_parts || rank < 0 ||
      rank >= nranks)
    return fail(c, MAD_ERR_INVALID_ARG, "nranks, row_begin, x_parts or rank");
  if (row_begin[0] != 0 || row_begin[nranks] != c->V)
    return fail(c, MAD_ERR_INVALID_ARG, "row_begin must run from 0 to V");
  for (int r = 0; r < nranks; ++r) {
    if (row_begin[r + 1] < row_begin[r])
      return fail(c, MAD_ERR_INVALID_ARG, "row_begin must not decrease");
    if (row_begin[r] % 32 != 0 && row_begin[r] != c->V)
      return fail(c, MAD_ERR_INVALID_ARG, "shard boundaries must be multiples of 32 rows");
    if (row_begin[r + 1] > row_begin[r] && !x_parts[r])
      return fail(c, MAD_ERR_INVALID_ARG, "x_parts of a non-empty shard is NULL");
  }
  if (t->mask & ~(uint32_t)(MAD_TERM_SPRING | MAD_TERM_INERTIA))
    return fail(c, MAD_ERR_UNIMPLEMENTED, "sharded evaluation takes spring and inertia terms");
  if (t->flags & (MAD_EVAL_EDGE_SCATTER | MAD_EVAL_PATCH_STAGED))
    return fail(c, MAD_ERR_UNIMPLEMENTED, "sharded evaluation uses the row kernel");
  if (c->active >= 0)
    return fail(c, MAD_ERR_UNIMPLEMENTED, "sharded evaluation needs the mesh pattern (no pairs)");
  if (!c->rows_cslots)
    return fail(c, MAD_ERR_UNIMPLEMENTED, "sharded evaluation needs compact row tables");
  const int lo = row_begin[rank], hi = row_begin[rank + 1];
  if (hi > lo && (!g_part || !H_part))
    return fail(c, MAD_ERR_INVALID_ARG, "g_part and H_part must be device pointers");
  const int64_t block_lo = c->rp_host[lo];
  cudaError_t e = launch_rows_eval_shard(rows_launch(c), *t, nranks, row_begin, block_lo,
                                         x_parts, rank, g_part, H_part, energy,
                                         as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(c, e, "mad_eval_shard launch");
  return MAD_OK;
}

mad_status mad_add_pairs(mad_ctx* c, int32_t n, const int32_t* ij, const void* rest,
                         void* stream) {
  if (!c) return MAD_ERR_INVALID_ARG;
  if (n < 0) return fail(c, MAD_ERR_INVALID_ARG, "n < 0");
  if (n > c->max_pairs) return fail(c, MAD_ERR_CAPACITY, "n exceeds max_pairs");
  c->vfs.n = -1;  // a new pair set drops the installed vertex-face terms
  if (n == 0) {
    c->active = -1;  // the mesh pattern, no pairs
    return MAD_OK;
  }
  if (!ij || !rest) return fail(c, MAD_ERR_INVALID_ARG, "ij and rest must be device pointers");
  const int next = c->active < 0 ? 0 : 1 - c->active;
  PairLaunch L;
  L.V = c->V;
  L.dtype = c->dtype;
  L.capacity = c->capacity;
  L.nnzb_base = c->nnzb_base;
  L.max_pairs = c->max_pairs;
  L.base_rp = c->pat.rp;
  L.base_ci = c->pat.ci;
  L.cnt = c->cnt;
  L.tsum = c->tsum;
  L.newcnt = c->newcnt;
  L.pe_pid = c->pe_pid;
  L.status = c->status;
  L.base_nnzb_dev = c->base_nnzb_dev;
  const DynBuf* prev = c->active < 0 ? nullptr : &c->buf[c->active];
  cudaError_t e = launch_add_pairs(L, n, ij, rest, c->buf[next], prev, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(c, e, "mad_add_pairs launch");
  c->active = next;
  return MAD_OK;
}

mad_status mad_add_vf(mad_ctx* c, int32_t n, const int32_t* vf, void* stream) {
  if (!c) return MAD_ERR_INVALID_ARG;
  if (n < 0) return fail(c, MAD_ERR_INVALID_ARG, "n < 0");
  if (n > c->vfs.max_terms)
    return fail(c, MAD_ERR_CAPACITY, "n exceeds max_pairs / 3 vertex-face terms");
  if (n > 0 && !vf) return fail(c, MAD_ERR_INVALID_ARG, "vf must be a device pointer");
  if (c->dof != 3) return fail(c, MAD_ERR_UNIMPLEMENTED, "vertex-face terms need dof 3");
  cudaStream_t s = as_stream(stream);
  cudaError_t e = launch_vf_install_expand(c->vfs, n, vf, c->V, c->F_dev, c->nF, s);
  if (e != cudaSuccess) return cuda_fail(c, e, "mad_add_vf launch");
  // the terms' (vertex, corner) pairs become the pair set
  mad_status st = mad_add_pairs(c, 3 * n, c->vfs.pairs, c->vfs.zero_rest, stream);
  if (st != MAD_OK) return st;
  const int32_t* rp = c->active < 0 ? c->pat.rp : c->buf[c->active].rp;
  const int32_t* ci = c->active < 0 ? c->pat.ci : c->buf[c->active].ci;
  e = launch_vf_install_tables(c->vfs, n, c->V, c->F_dev, c->nF, rp, ci, c->cnt, c->status, s);
  if (e != cudaSuccess) return cuda_fail(c, e, "mad_add_vf tables");
  c->vfs.n = n;
  return MAD_OK;
}

namespace {
mad_status jac_mask_ok(const mad_ctx* c, uint32_t mask, std::string* why) {
  const uint32_t known = MAD_TERM_SPRING | MAD_TERM_INERTIA | MAD_TERM_SYMDIR | MAD_TERM_PAIR |
                         MAD_TERM_AREA | MAD_TERM_ARAP | MAD_TERM_VF;
  if (mask & ~known) {
    *why = "unknown term bits in mask";
    return MAD_ERR_INVALID_ARG;
  }
  if (mask & (MAD_TERM_PAIR | MAD_TERM_AREA | MAD_TERM_ARAP | MAD_TERM_VF)) {
    *why = "pair, area, ARAP and vertex-face terms are not part of the vector-valued objective";
    return MAD_ERR_UNIMPLEMENTED;
  }
  if ((mask & MAD_TERM_SYMDIR) && c->dof != 2) {
    *why = "symmetric Dirichlet term needs dof 2";
    return MAD_ERR_UNIMPLEMENTED;
  }
  return MAD_OK;
}
}  // namespace

mad_status mad_jacobian_shape(const mad_ctx* c, uint32_t mask, int64_t* nrows, int64_t* nnz) {
  if (!c || !nrows || !nnz) return MAD_ERR_INVALID_ARG;
  std::string why;
  const mad_status st = jac_mask_ok(c, mask, &why);
  if (st != MAD_OK) return st;
  jac_shape(c->V, c->dof, mask, c->E, c->nF, nrows, nnz);
  return MAD_OK;
}

mad_status mad_jacobian_pattern(mad_ctx* c, uint32_t mask, int64_t* row_ptr, int32_t* col_idx,
                                void* stream) {
  if (!c) return MAD_ERR_INVALID_ARG;
  std::string why;
  const mad_status st = jac_mask_ok(c, mask, &why);
  if (st != MAD_OK) return fail(c, st, why);
  int64_t rows = 0, nnz = 0;
  jac_shape(c->V, c->dof, mask, c->E, c->nF, &rows, &nnz);
  if (!row_ptr || (nnz > 0 && !col_idx))
    return fail(c, MAD_ERR_INVALID_ARG, "row_ptr and col_idx must be device pointers");
  const cudaError_t e = launch_jac_pattern(c->V, c->dof, mask, c->E, c->pat.edges, c->nF,
                                           c->F_dev, row_ptr, col_idx, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(c, e, "mad_jacobian_pattern launch");
  return MAD_OK;
}

mad_status mad_jacobian(mad_ctx* c, const void* x, const mad_terms* t, void* r, void* J_vals,
                        void* stream) {
  if (!c) return MAD_ERR_INVALID_ARG;
  if (!t) return fail(c, MAD_ERR_INVALID_ARG, "terms is NULL");
  std::string why;
  const mad_status st = jac_mask_ok(c, t->mask, &why);
  if (st != MAD_OK) return fail(c, st, why);
  if ((t->mask & MAD_TERM_SPRING) && c->E > 0 && !t->spring_rest)
    return fail(c, MAD_ERR_INVALID_ARG, "spring term active but spring_rest is NULL");
  if ((t->mask & MAD_TERM_INERTIA) && c->V > 0 && !t->inertia_xt)
    return fail(c, MAD_ERR_INVALID_ARG, "inertia term active but inertia_xt is NULL");
  if ((t->mask & MAD_TERM_SYMDIR) && c->nF > 0 && (!t->face_Minv || !t->face_area))
    return fail(c, MAD_ERR_INVALID_ARG, "symmetric Dirichlet term needs face_Minv and face_area");
  int64_t rows = 0, nnz = 0;
  jac_shape(c->V, c->dof, t->mask, c->E, c->nF, &rows, &nnz);
  if (rows > 0 && (!x || !r || !J_vals))
    return fail(c, MAD_ERR_INVALID_ARG, "x, r and J_vals must be device pointers");
  const cudaError_t e = launch_jacobian(c->dtype, c->V, c->dof, t->mask, c->E, c->pat.edges,
                                        c->nF, c->F_dev, *t, x, r, J_vals, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(c, e, "mad_jacobian launch");
  return MAD_OK;
}

mad_status mad_status_sync(mad_ctx* c, void* stream) {
  if (!c) return MAD_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(c, e, "mad_status_sync");
  int32_t st = 0;
  e = cudaMemcpy(&st, c->status, sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(c, e, "mad_status_sync read");
  e = cudaMemset(c->status, 0, sizeof(int32_t));
  if (e != cudaSuccess) return cuda_fail(c, e, "mad_status_sync clear");
  if (st & kStatusCapacity)
    return fail(c, MAD_ERR_CAPACITY, "pair blocks exceeded the CSR capacity");
  if (st & kStatusIndex)
    return fail(c, MAD_ERR_INDEX, "a pair had an index out of range or i == j");
  if (st & kStatusTimeout) return fail(c, MAD_ERR_TIMEOUT, "a device wait timed out");
  return MAD_OK;
}

mad_status mad_eval_host(mad_ctx* c, const void* x, const mad_terms* t, void* g,
                         void* H_vals, double* energy, void* stream) {
  if (!c) return MAD_ERR_INVALID_ARG;
  if (c->V > 0 && (!x || !g || !H_vals))
    return fail(c, MAD_ERR_INVALID_ARG, "x, g and H_vals must be host pointers");
  cudaStream_t s = as_stream(stream);
  const size_t vb = (size_t)c->V * c->dof * c->esz;
  const size_t hb = (size_t)c->capacity * c->dof * c->dof * c->esz;
  cudaError_t e;
  if (!c->hx) {
    if ((e = cudaMalloc(&c->hx, vb ? vb : 16)) != cudaSuccess ||
        (e = cudaMalloc(&c->hg, vb ? vb : 16)) != cudaSuccess ||
        (e = cudaMalloc(&c->hH, hb ? hb : 16)) != cudaSuccess ||
        (e = cudaMalloc(&c->he, sizeof(double))) != cudaSuccess)
      return cuda_fail(c, e, "mad_eval_host staging");
  }
  int32_t nnzb = c->nnzb_base;
  if (c->active >= 0) {
    if ((e = cudaMemcpyAsync(&nnzb, c->buf[c->active].nnzb, sizeof(int32_t),
                             cudaMemcpyDeviceToHost, s)) != cudaSuccess)
      return cuda_fail(c, e, "mad_eval_host nnzb");
  }
  if (vb && (e = cudaMemcpyAsync(c->hx, x, vb, cudaMemcpyHostToDevice, s)) != cudaSuccess)
    return cuda_fail(c, e, "mad_eval_host x");
  mad_status st = mad_eval(c, c->hx, t, c->hg, c->hH, energy ? c->he : nullptr, stream);
  if (st != MAD_OK) return st;
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(c, e, "mad_eval_host");
  const size_t hcopy = (size_t)nnzb * c->dof * c->dof * c->esz;
  if (vb && (e = cudaMemcpyAsync(g, c->hg, vb, cudaMemcpyDeviceToHost, s)) != cudaSuccess)
    return cuda_fail(c, e, "mad_eval_host g");
  if (hcopy && (e = cudaMemcpyAsync(H_vals, c->hH, hcopy, cudaMemcpyDeviceToHost, s)) != cudaSuccess)
    return cuda_fail(c, e, "mad_eval_host H");
  if (energy &&
      (e = cudaMemcpyAsync(energy, c->he, sizeof(double), cudaMemcpyDeviceToHost, s)) != cudaSuccess)
    return cuda_fail(c, e, "mad_eval_host energy");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(c, e, "mad_eval_host");
  return MAD_OK;
}

const char* mad_last_error(const mad_ctx* c) {
  if (!c) return g_create_error.c_str();
  return c->err.c_str();
}

void mad_destroy(mad_ctx* c) { free_ctx(c); }

mad_status mad_selftest_dual(int32_t n, const double* ab, double* out) {
  if (n < 0 || (n > 0 && (!ab || !out))) return MAD_ERR_INVALID_ARG;
  if (n == 0) return MAD_OK;
  double *dab = nullptr, *dout = nullptr;
  cudaError_t e = cudaMalloc(&dab, sizeof(double) * 2 * n);
  if (e == cudaSuccess) e = cudaMalloc(&dout, sizeof(double) * 24 * n);
  if (e == cudaSuccess) e = cudaMemcpy(dab, ab, sizeof(double) * 2 * n, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = selftest_dual(n, dab, dout);
  if (e == cudaSuccess) e = cudaMemcpy(out, dout, sizeof(double) * 24 * n, cudaMemcpyDeviceToHost);
  cudaFree(dab);
  cudaFree(dout);
  if (e != cudaSuccess) {
    g_create_error = std::string("mad_selftest_dual: ") + cudaGetErrorString(e);
    return MAD_ERR_CUDA;
  }
  return MAD_OK;
}

}  // extern "C"
