// mad_internal.h -- structures shared by the host side of libmad and its
// kernels.  Nothing here is part of the public C ABI (include/mad.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "../../include/mad.h"

namespace mad {

// One patch = a set of OWNED vertices (each vertex is owned by exactly one
// patch) plus the ribbon: every vertex outside the set that shares a term with
// it.  A patch evaluates every term touching one of its owned vertices and
// writes only the rows of its owned vertices, so no two CUDA blocks ever
// write the same Hessian block or gradient row (page "Locality-Aware
// Automatic Differentiation on the GPU for Mesh-Based Computations", section
// 方法, key design 2: one CUDA block per patch, ribbon elements cache the
// cross-patch neighbours).
struct PatchHdr {
  int32_t vbeg, nv, no, nstage;  // local vertices [vbeg, vbeg+nv), owned first;
                                 // nstage = base blocks of the owned rows
  int32_t ebeg, ne, ecbeg, nce;  // edge terms; colour c spans
                                 // ecol[ecbeg+c] .. ecol[ecbeg+c+1] (relative)
  int32_t fbeg, nf, fcbeg, ncf;  // face terms, same layout
  int32_t sbeg, stride;  // row slots: owned row r's slot p is sbeg + r*stride + p
  int32_t rbeg, nruns;   // runs of consecutive owned vertices: runs[rbeg .. +nruns)
};

// Block-offset lookup for an edge term (built once per topology): local
// indices of its two vertices and, for each owned endpoint, the position of
// the other endpoint's column inside that endpoint's (mesh-pattern) row.
// kNotOwned marks an endpoint that belongs to another patch.
struct EdgeLut {
  uint16_t la, lb, pab, pba;
};

// Face-term lookup: local vertex indices and pos[k][m] = position of column
// F[m] in the row of corner k (kNotOwned when corner k is not owned).
struct FaceLut {
  uint16_t l[3];
  uint16_t pos[3][3];
  int32_t fid;
};

constexpr uint16_t kNotOwned = 0xFFFF;
constexpr uint16_t kNoSlot = 0xFFFF;

// Pair entry position word: low 30 bits = block position inside the row of
// the current (dynamic) pattern; bit 30 set when this entry created that
// block (first entry of its column and the column is not in the mesh row).
constexpr int32_t kPairNewBlock = 1 << 30;
constexpr int32_t kPairPosMask = (1 << 30) - 1;
constexpr uint32_t kPmaskOverflow = 1u << 31;

// Per-owned-vertex meta: x = mesh-pattern row length | diagonal position << 16,
// y = first row of the vertex's run | run index << 16.  A run is a maximal
// sequence of owned vertices with consecutive ids; their Hessian rows are
// consecutive in H, so a run is staged and written back as one piece.
__host__ __device__ inline uint32_t pack_meta(int blen, int dpos) {
  return (uint32_t)blen | ((uint32_t)dpos << 16);
}

// Row slots (the gather form of the block-offset lookup): for every block of
// an owned row of the mesh pattern, in column order, the local index of the
// column's vertex and the id of the edge joining it to the row's vertex (-1
// on the diagonal); rows are padded to the patch's stride with kNoSlot.

// Device status bits (sticky; read by mad_status_sync).
enum : int32_t { kStatusIndex = 1, kStatusCapacity = 2, kStatusTimeout = 4 };

struct HostPatches {
  std::vector<PatchHdr> hdr;
  std::vector<int32_t> vgid;
  std::vector<uint2> meta;      // indexed like vgid (owned entries used)
  std::vector<EdgeLut> elut;
  std::vector<int32_t> eid;
  std::vector<int32_t> ecol;
  std::vector<FaceLut> flut;
  std::vector<int32_t> fcol;
  std::vector<uint16_t> slot_lidx;
  std::vector<int32_t> slot_eid;
  std::vector<uint32_t> runs;  // first row | row count << 16
  int nv_max = 0, no_max = 0;
  int slots_max = 0;  // most row slots (owned rows x stride) of one patch
};

// Host partitioner (partition.cpp).  rp/ci: mesh pattern (host copies).
// Returns "" on success, else an error message.
std::string build_patches(int V, int nF, const int32_t* F, const int32_t* rp,
                          const int32_t* ci, const double* xyz, int xyz_dim,
                          int target_owned, int max_stage_blocks,
                          HostPatches& out);

// Row tables of the row-streaming assembly kernel (rows.cu): warp w owns
// rows 32w .. 32w+31.  For every row, its off-diagonal mesh-pattern blocks in
// column order: the column vertex and the id of the edge joining it to the
// row's vertex.  The first `s0` of them are stored slot-major per tile of 32
// rows (slot k of row 32t+l at (t*s0 + k)*32 + l, so a warp's loads are
// coalesced); further ones (rows longer than s0) in an overflow table.
struct HostRowTables {
  int s0 = 0;
  std::vector<int2> slots;        // [ntiles][s0][32] {col, eid}, {-1,-1} empty
  std::vector<uint32_t> meta;     // [V] off-diagonal count | diagonal position << 16
  std::vector<int32_t> ofl_ptr;   // [V+1] overflow slots per row (prefix sums)
  std::vector<int2> ofl;          // overflow slots
  // Compact form of the same slots, built when every delta below fits 16
  // bits (empty vectors otherwise).  Per tile t of 32 rows: ctile[t] =
  // {row_ptr of row 32t, id of the first edge (a, b) with a >= 32t, mask of
  // the tile's rows that continue in the overflow table, 0}.  Per slot: the
  // column minus the row and the edge id minus the tile's first edge id, as
  // two int16 halves (low, high) of one word; 0 marks an empty slot (a
  // column never equals its row).  Row pointers follow from the tile's
  // row_ptr and the rows' lengths, so neither row_ptr nor meta is read.
  std::vector<int4> ctile;        // [ntiles]
  std::vector<uint32_t> cslots;   // [ntiles][s0][32]
};
std::string build_row_tables(int V, const int32_t* rp, const int32_t* ci, int s0_cap,
                             HostRowTables& out);

// Face rows of the same kernel: for every row i, the faces that have vertex i
// as a corner, in face order.  Entry {f, j, k, c | pj << 2 | pk << 17}: i is
// corner c of face f, j and k are corners c+1 and c+2 (mod 3), pj and pk the
// block positions of columns j and k in row i of the mesh pattern.  The first
// `sf` entries of a row are stored slot-major per tile of 32 rows, like the
// edge slots; the rest in an overflow table, and then the row's last slot has
// the sign bit of k set.  Rows of 32768 blocks or more do
// not fit the 15-bit positions: the builder then returns an error and the
// face terms stay on the patch kernel.
constexpr int kFaceRowSlots = 6;
constexpr int kFacePosBits = 15;
struct HostFaceRows {
  int sf = 0;
  std::vector<int4> slots;       // [ntiles][sf][32], f = -1 empty
  std::vector<int32_t> ofl_ptr;  // [V+1]
  std::vector<int4> ofl;
  // the same incidences as 3f + c only (the Hessian-vector product reads
  // per-face corner results): -1 empty; bit 31 set on the last slot of a row
  // that continues in the overflow table
  std::vector<int32_t> cslots;   // [ntiles][sf][32]
  std::vector<int32_t> cofl;     // overflow, same order as ofl
};
std::string build_face_rows(int V, int nF, const int32_t* F, const int32_t* rp,
                            const int32_t* ci, HostFaceRows& out);

// ---- dynamic pattern buffers ------------------------------------------
struct DynBuf {
  int32_t* rp = nullptr;      // [V+1]
  int32_t* ci = nullptr;      // [capacity]
  int32_t* nnzb = nullptr;    // [1]
  int32_t* prow = nullptr;    // [V+1] pair entries per row (exclusive scan)
  int32_t* pe_col = nullptr;  // [2*max_pairs] partner vertex, sorted per row
  int32_t* pe_pos = nullptr;  // [2*max_pairs] position word (see above)
  void* pe_rest = nullptr;    // [2*max_pairs] rest length (dtype)
  // [V] per row: bit p set when merged position p (< 31) holds an inserted
  // block; kPmaskOverflow | count when an inserted position is 31 or more
  uint32_t* pmask = nullptr;
};

// vertex-face terms (vf.cu): the active pattern, the terms and positions
struct VfLaunch {
  int n = 0, V = 0, nF = 0;
  const int32_t* vf = nullptr;
  const void* rest = nullptr;
  double k = 0.0;
  const int32_t* F = nullptr;
  const void* x = nullptr;
  const int32_t* rp = nullptr;
  const int32_t* ci = nullptr;
  int32_t* status = nullptr;
  bool generic = false;  // the energy as a plain expression (MAD_EVAL_GENERIC_AD)
};
cudaError_t launch_vf_eval(int dtype, const VfLaunch& L, void* g, void* H, double* energy,
                           cudaStream_t s);
// An installed vertex-face term set (mad_add_vf): the terms, their pairs for
// the insertion and the per-row incidence tables of the gather form (vf.cu).
struct VfSet {
  int max_terms = 0;        // largest set (max_pairs / 3)
  int n = -1;               // installed terms; -1: none installed
  int32_t* terms = nullptr; // [max_terms][2] (vertex p, face f)
  int32_t* pairs = nullptr; // [3 max_terms][2] (p, corner) for the insertion
  void* zero_rest = nullptr;// [3 max_terms] zeros in the dtype (rest of those pairs)
  int32_t* vrow = nullptr;  // [V+1] incidences per row (exclusive scan)
  int32_t* ent = nullptr;   // [4 max_terms][8] entries (see vf.cu)
  int32_t* scan_tmp = nullptr;
  int32_t* vslot = nullptr; // [max_terms][4] entry index of each (term, role)
  void* rec = nullptr;      // [4 max_terms][40] per-entry shares written by the term pass
  double* epart = nullptr;  // [ceil(max_terms / 256)] per-block energy of the term pass
};
cudaError_t launch_vf_install_expand(const VfSet& S, int n, const int32_t* vf, int V,
                                     const int32_t* F, int nF, cudaStream_t s);
cudaError_t launch_vf_install_tables(const VfSet& S, int n, int V, const int32_t* F, int nF,
                                     const int32_t* rp, const int32_t* ci, int32_t* cnt,
                                     int32_t* status, cudaStream_t s);
cudaError_t launch_vf_rows_eval(int dtype, const VfSet& S, const VfLaunch& L, void* g, void* H,
                                double* energy, cudaStream_t s);
// the term pass alone: one record per installed term (S.rec), for the row
// kernel to gather
cudaError_t launch_vf_term_pass(int dtype, const VfSet& S, const VfLaunch& L, cudaStream_t s);
cudaError_t launch_vf_rows_hvp(int dtype, const VfSet& S, const VfLaunch& L, const void* v,
                               void* y, cudaStream_t s);
cudaError_t launch_vf_hvp(int dtype, const VfLaunch& L, const void* v, void* y, cudaStream_t s);

// ---- launchers (defined in the .cu files) ------------------------------
// scan.cu: exclusive scan of n int32 values in -> out[0..n], out[n] = total.
// tmp must hold scan_tmp_elems(n) ints.
size_t scan_tmp_elems(int64_t n);
cudaError_t scan_exclusive(const int32_t* in, int32_t* out, int64_t n,
                           int32_t* tmp, cudaStream_t s);

// topology.cu
struct PatternDev {
  int32_t* rp;      // [V+1]
  int32_t* ci;      // [nnzb]
  int32_t* diag;    // [V]
  int32_t* edges;   // [E][2]
  int32_t nnzb, E;
};
// Builds the mesh pattern and the sorted edge list; allocates the outputs
// with cudaMalloc.  Returns "" or an error message.
std::string build_pattern_gpu(int V, int nF, const int32_t* F_dev,
                              cudaStream_t s, PatternDev& out);

// eval.cu
struct EvalLaunch {
  int dtype, dof, n_patches, nv_max, no_max, slots_max;
  int grid;       // persistent blocks of the assembly kernel (0 = one per patch)
  int stage_cap;  // staging capacity in elements of the dtype
  const PatchHdr* hdr;
  const int32_t* vgid;
  const uint2* meta;
  const uint32_t* runs;
  const EdgeLut* elut;
  const int32_t* eid;
  const int32_t* ecol;
  const FaceLut* flut;
  const int32_t* fcol;
  const uint16_t* slot_lidx;
  const int32_t* slot_eid;
  int rho;            // staging room per row for inserted pair blocks
  const int32_t* rp;  // active row_ptr
  // pairs (active set); prow == nullptr when no pairs are active
  const int32_t* prow;
  const int32_t* pe_col;
  const int32_t* pe_pos;
  const void* pe_rest;
  double* epart;  // [n_patches]
};
size_t eval_smem_bytes(const EvalLaunch& L, bool hvp);
// persistent grid of the assembly kernel for this launch's shared memory
int eval_grid(const EvalLaunch& L);
// staging elements one patch needs with `rho` spare blocks per row
size_t patch_stage_elems(const PatchHdr& h, int dof, int esz, int rho);
cudaError_t launch_eval(const EvalLaunch& L, const mad_terms& t, const void* x,
                        void* g, void* H, double* energy, cudaStream_t s);
cudaError_t launch_hvp(const EvalLaunch& L, const mad_terms& t, const void* x,
                       const void* v, void* y, cudaStream_t s);
cudaError_t eval_set_smem_limits(int dtype, int dof, size_t bytes);

// pairs.cu
struct PairLaunch {
  int V, dtype, capacity, nnzb_base, max_pairs;
  const int32_t* base_rp;
  const int32_t* base_ci;
  int32_t* cnt;     // [V+1] pair entries per row; zero between calls
  int32_t* tsum;    // [pair_scratch_elems(V)] per-block and per-tile counts;
                    // zero at creation
  int32_t* newcnt;  // [V+1] new blocks per row
  int32_t* pe_pid;  // [2*max_pairs]
  int32_t* status;  // device status word
  const int32_t* base_nnzb_dev;  // [1] block count of the mesh pattern
};
// int32 scratch of the insertion kernels (block and tile counts)
size_t pair_scratch_elems(int V);
cudaError_t launch_add_pairs(const PairLaunch& L, int n, const int32_t* ij,
                             const void* rest, const DynBuf& nb,
                             const DynBuf* prev /* nullptr = mesh pattern */,
                             cudaStream_t s);

// rows.cu
struct RowsLaunch {
  int dtype, dof, V, s0, rho;
  int sf;                  // face slots per row (0: no face rows)
  const int4* fslots;
  const int32_t* fofl_ptr;
  const int4* fofl;
  const int32_t* fcslots;  // incidences as 3f + c (see HostFaceRows)
  const int32_t* fcofl;
  int nF;
  const int32_t* F;        // [nF][3]
  void* fhv;               // [nF][3][2] per-face corner results of H v (scratch)
  const int2* slots;
  const uint32_t* meta;
  const int32_t* ofl_ptr;
  const int2* ofl;
  const int4* ctile;        // compact slots (see HostRowTables); nullptr if absent
  const uint32_t* cslots;
  const int32_t* rp;  // active row_ptr
  const int32_t* prow;
  const int32_t* pe_col;
  const int32_t* pe_pos;
  const void* pe_rest;
  const uint32_t* pmask;  // inserted positions per row (DynBuf::pmask)
  // [2*max_pairs][4] per pair entry: the partner's position (DOF values,
  // zero padded) and the rest length in the last value; scratch the compact
  // row kernel fills before each assembly with pairs
  void* pe_xr = nullptr;
  double* epart;  // [rows_blocks(V)]
  // installed vertex-face terms gathered into the rows (nullptr: none)
  const int32_t* vrow = nullptr;
  const int32_t* vent = nullptr;
  const void* vrec = nullptr;
};
int rows_blocks(int V);
size_t rows_smem_bytes(const RowsLaunch& L);
cudaError_t rows_set_smem_limits(int dtype, int dof, size_t bytes);
cudaError_t launch_rows_eval(const RowsLaunch& L, const mad_terms& t, const void* x, void* g,
                             void* H, double* energy, cudaStream_t s);
cudaError_t launch_rows_hvp(const RowsLaunch& L, const mad_terms& t, const void* x,
                            const void* v, void* y, cudaStream_t s);
// the rows of one shard (edge and vertex terms, compact row tables)
cudaError_t launch_rows_eval_shard(const RowsLaunch& L, const mad_terms& t, int nranks,
                                   const int32_t* row_begin, int64_t block_lo,
                                   const void* const* x_parts, int rank, void* g, void* H,
                                   double* energy, cudaStream_t s);

// jacobian.cu
void jac_shape(int V, int dof, unsigned mask, int nE, int nF, int64_t* rows, int64_t* nnz);
cudaError_t launch_jac_pattern(int V, int dof, unsigned mask, int nE, const int32_t* edges,
                               int nF, const int32_t* F, int64_t* rp, int32_t* ci,
                               cudaStream_t s);
cudaError_t launch_jacobian(int dtype, int V, int dof, unsigned mask, int nE,
                            const int32_t* edges, int nF, const int32_t* F, const mad_terms& t,
                            const void* x, void* r, void* J, cudaStream_t s);

// selftest.cu
cudaError_t selftest_dual(int n, const double* ab_dev, double* out_dev);

}  // namespace mad
