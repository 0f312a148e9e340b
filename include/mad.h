/*
 * mad.h -- C ABI of the B200 mesh-autodiff assembly library (libmad.so).
 *
 * The library implements the data-parallel hot path described on the page
 * "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
 * Computations" (reading note), section 方法 (method):
 *   * a scalar objective F(x) = sum_j f_j(x_j) of local terms on a triangle
 *     mesh, each term depending on a small fixed stencil x_j;
 *   * per-term forward-mode automatic differentiation giving the dense local
 *     gradient g_j and Hessian H_j in registers (key design 1);
 *   * assembly g = sum_j S_j^T g_j and H = sum_j S_j^T H_j S_j into a global
 *     gradient and a block-CSR Hessian whose pattern is preallocated from
 *     mesh topology by a parallel count + prefix sum (key design 3), with
 *     the mesh processed patch by patch, one CUDA block per patch, and
 *     ribbon (ghost) vertices around each patch (key design 2);
 *   * runtime vertex-vertex interaction pairs inserted into a double-
 *     buffered CSR with reserved slack, entirely on the GPU (key design 4);
 *   * a matrix-free Hessian-vector product (section 实验结果 (results), the
 *     parameterization application).
 *
 * Conventions shared by every entry point
 *   - Pointers documented "device" are CUDA device pointers in the current
 *     device's memory; "host" pointers are ordinary CPU memory.
 *   - Floating-point arrays use the context's dtype (MAD_F32 -> float,
 *     MAD_F64 -> double); `energy` outputs are always double.
 *   - Positions, gradients and vectors are [V][dof] interleaved (dof = 2 or 3).
 *   - The Hessian is block CSR with b x b blocks, b = dof: both triangles
 *     stored, 0-based int32 row_ptr/col_idx, columns strictly ascending in a
 *     row, the diagonal block always present, blocks contiguous and row-major
 *     inside a block: element (r, c) of block q is H_vals[q*b*b + r*b + c].
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call after mad_create is stream-ordered, performs no
 *     host synchronisation and allocates no memory.
 *   - Synchronous argument errors are returned at once and nothing is
 *     launched.  Errors found on the device (a pair index out of range, CSR
 *     capacity exceeded) are recorded in a sticky device status word and are
 *     reported by mad_status_sync(); no kernel traps or asserts.
 *   - A context is used by one host thread at a time, and its calls are
 *     issued on one stream (or streams ordered by events): the context keeps
 *     per-call device scratch (per-face product results, the gathered pair
 *     partner positions, the vertex-face shares, energy partials) that two
 *     calls running at once on unordered streams would share.
 */
#ifndef MAD_H_
#define MAD_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct mad_ctx mad_ctx; /* opaque, owned by the library */

typedef enum {
  MAD_OK = 0,
  MAD_ERR_INVALID_ARG = 1,   /* bad pointer, size, index, dtype or mask      */
  MAD_ERR_CUDA = 2,          /* a CUDA runtime call failed (see last_error)  */
  MAD_ERR_OOM = 3,           /* device or host allocation failed (create)    */
  MAD_ERR_CAPACITY = 4,      /* pairs or CSR blocks exceed reserved capacity */
  MAD_ERR_INDEX = 5,         /* device-detected index out of range           */
  MAD_ERR_TIMEOUT = 6,       /* a bounded device wait gave up                */
  MAD_ERR_UNIMPLEMENTED = 7, /* term / dof / dtype combination not built     */
  MAD_ERR_STATE = 8          /* call not valid in the context's state        */
} mad_status;

typedef enum { MAD_F32 = 0, MAD_F64 = 1 } mad_dtype;

/* Local energy terms (bit mask).  Section 方法 states the model (local
 * terms on vertices, edges, faces and runtime pairs); the concrete energies
 * are the applications' (section 实验结果): mass-spring cloth and the
 * parameterization energy.                                                  */
enum {
  MAD_TERM_SPRING = 1u,  /* per mesh edge: 1/2 k (|xi - xj| - L0_e)^2         */
  MAD_TERM_INERTIA = 2u, /* per vertex: 1/2 w |xi - xt_i|^2                   */
  MAD_TERM_SYMDIR = 4u,  /* per face, dof 2: A_f (|J|_F^2 + |J^-1|_F^2),
                            J = [u1-u0, u2-u0] Minv_f                         */
  MAD_TERM_PAIR = 8u,    /* per runtime pair: 1/2 k_p (|xi - xj| - r_p)^2     */
  MAD_TERM_AREA = 16u,   /* per face, dof 3 (a 9-variable stencil): area
                            preservation 1/2 k_a (A_f - A0_f)^2 / A0_f with
                            A_f = |(x1-x0) x (x2-x0)| / 2, A0_f = face_area */
  MAD_TERM_ARAP = 32u,   /* per face, dof 2: as-rigid-as-possible
                            A_f |J - R(J)|_F^2, J as for MAD_TERM_SYMDIR
                            (same face_Minv and face_area), R(J) the closest
                            rotation.  With MAD_TERM_SYMDIR both energies
                            are summed per face.  Needs det J > 0 (the
                            closest rotation is unique there).              */
  MAD_TERM_VF = 64u      /* per vertex-face term (dof 3): 1/2 k_c (d - r)^2,
                            d the signed distance of vertex p to the plane of
                            face f (n = (x1-x0) x (x2-x0)).  Either install
                            the terms with mad_add_vf and pass t->vf = NULL
                            (gathered per row: reproducible), or insert the
                            pairs (p, corner) of every term with
                            mad_add_pairs and pass the terms in t->vf (one
                            thread per term adds with atomics, so the
                            blocks are not bit-reproducible across runs).
                            Not with MAD_TERM_PAIR (its pair list would hold
                            those pairs too).                               */
};

/* Evaluation flags. */
enum {
  /* Seed forward-mode tangents on every stencil DOF (width 2*dof per edge or
   * pair term, 3*dof per face term) instead of the default, which seeds the
   * term's natural variables (the edge vector; the 2x2 Jacobian J) and maps
   * g_j, H_j back through the term's constant linear input map.  Both give
   * the same derivatives up to rounding.                                     */
  MAD_EVAL_FULL_STENCIL_AD = 1u,
  /* Assemble edge terms by scattering each term once into the rows of its
   * owned endpoints, colour by colour, instead of the default, where the
   * thread that owns a row gathers the derivatives of the row's edge terms
   * (each term evaluated once per owned endpoint).  Same results up to
   * rounding; provided for comparison.                                       */
  MAD_EVAL_EDGE_SCATTER = 2u,  /* (not with MAD_TERM_AREA or MAD_TERM_ARAP) */
  /* Use the patch kernel (one CUDA block per patch, positions of the patch's
   * owned and ribbon vertices staged in shared memory) instead of the
   * default row-streaming kernel (one warp per 32 consecutive rows, no
   * block-wide barriers).  Same results up to rounding.  The patch kernel
   * does not evaluate MAD_TERM_AREA or MAD_TERM_ARAP (MAD_ERR_UNIMPLEMENTED). */
  MAD_EVAL_PATCH_STAGED = 4u,
  /* Differentiate every energy as written: the spring and pair, symmetric
   * Dirichlet, area-preservation and vertex-face energies as plain
   * expressions (square roots, products, 1/det), each differentiated by the
   * AD number types' own operations and elementary functions, instead of
   * the default, which evaluates each as a univariate function of one AD
   * intermediate with that function's first and second derivatives written
   * out (one chain-rule step).  Same derivatives up to rounding; the default
   * is faster.  Not with MAD_EVAL_FULL_STENCIL_AD (MAD_ERR_INVALID_ARG), nor
   * with the patch kernel (MAD_ERR_UNIMPLEMENTED).                          */
  MAD_EVAL_GENERIC_AD = 8u
};

typedef struct {
  int32_t patch_faces;   /* target faces per patch; default 512           */
  float slack;           /* reserved CSR blocks beyond the mesh pattern, as a
                            fraction of its block count; default 0.10      */
  int32_t max_pairs;     /* largest pair set mad_add_pairs accepts; default
                            = reserved blocks / 2, at least 1024           */
  const double* part_xyz;/* optional host [V][part_dim] positions used only
                            to shape patches (Morton order); NULL = shape
                            patches by breadth-first growth on the graph   */
  int32_t part_dim;      /* 2 or 3 when part_xyz is given                  */
  int32_t smem_budget;   /* bytes of shared memory per CUDA block for the
                            staged Hessian rows; 0 = library default       */
} mad_opts;

/* Term parameters for one evaluation.  All arrays are device pointers in the
 * context's dtype, owned by the caller, read during the call only.         */
typedef struct {
  uint32_t mask;            /* MAD_TERM_* bits                               */
  uint32_t flags;           /* MAD_EVAL_* bits                               */
  const void* spring_rest;  /* [E] L0 per edge, in mad_edges() order         */
  double spring_k;          /* stiffness k                                   */
  const void* inertia_xt;   /* [V][dof] target positions xt                  */
  double inertia_w;         /* w = m / h^2                                   */
  const void* face_Minv;    /* [nF][2][2] row-major Dm^-1 per face (dof 2)   */
  const void* face_area;    /* [nF] rest area per face                       */
  double pair_k;            /* k_p for the current pair set                  */
  double area_k;            /* k_a of MAD_TERM_AREA                          */
  int32_t vf_n;             /* number of vertex-face terms (MAD_TERM_VF)     */
  const int32_t* vf;        /* [vf_n][2] (vertex p, face f) per term, or NULL
                               for the set installed by mad_add_vf          */
  const void* vf_rest;      /* [vf_n] rest offset r per term                 */
  double vf_k;              /* k_c of MAD_TERM_VF                            */
} mad_terms;

typedef struct {
  int32_t V, nF, E, dof;
  int32_t dtype;            /* mad_dtype                                     */
  int32_t nnzb_base;        /* blocks of the mesh pattern                    */
  int32_t capacity_blocks;  /* blocks the dynamic CSR can hold; H_vals must
                               hold capacity_blocks * dof * dof elements     */
  int32_t max_pairs;
  int32_t n_patches;
  int32_t max_patch_vertices;   /* owned + ribbon vertices of the largest patch */
  int32_t max_patch_owned;
  int32_t smem_bytes;       /* dynamic shared memory of the assembly kernel  */
  int64_t device_bytes;     /* device memory the context holds               */
  int32_t row_slot_bytes;   /* bytes per slot of the row tables that edge and
                               vertex terms on the mesh pattern read: 4 when
                               every column and edge id of a 32-row tile
                               lies within 16 bits of the row and of the
                               tile's first edge (bandwidth-ordered meshes),
                               else 8                                        */
} mad_info_t;

/* Fill *o with the defaults listed in mad_opts. */
void mad_default_opts(mad_opts* o);

/* Analyse the mesh and preallocate the block-CSR pattern (section 方法, key
 * design 3: the pattern follows from connectivity and the declared 1-ring
 * stencils; it is built on the GPU by a parallel per-row count, a prefix sum
 * and a fill, followed by a per-row sort).  Also extracts the unique edges,
 * partitions the vertices into patches (key design 2) and builds the
 * per-patch term tables and CSR block-offset lookup.
 *   V, nF   vertex and face counts (V >= 0, nF >= 0)
 *   F       HOST [nF][3] vertex indices; each in [0, V), three distinct
 *   dof     2 or 3;  dt  MAD_F32 or MAD_F64;  o  NULL for defaults
 *   out     receives the new context
 * Allocates all device memory the context will ever use and synchronises
 * `stream` once at the end.  Errors: MAD_ERR_INVALID_ARG (bad sizes or
 * faces), MAD_ERR_OOM, MAD_ERR_CUDA.  On error *out is NULL.               */
mad_status mad_create(int32_t V, int32_t nF, const int32_t* F, int32_t dof,
                      mad_dtype dt, const mad_opts* o, void* stream,
                      mad_ctx** out);

/* Sizes and layout facts of a context. */
mad_status mad_info(const mad_ctx* c, mad_info_t* info);

/* Unique undirected mesh edges (i < j) sorted by (i, j): DEVICE [E][2],
 * borrowed, valid until mad_destroy.  spring_rest is indexed in this order. */
mad_status mad_edges(const mad_ctx* c, const int32_t** ij, int32_t* E);

/* Current block-CSR pattern (the mesh pattern until the first
 * mad_add_pairs, then the pattern holding the latest pair set):
 * DEVICE row_ptr [V+1] and col_idx [capacity_blocks]; *nnzb_dev is a DEVICE
 * int32 holding the block count.  Borrowed; the pointers change with each
 * mad_add_pairs call (double buffering) and the contents are produced in
 * stream order.                                                          */
mad_status mad_pattern(const mad_ctx* c, const int32_t** row_ptr,
                       const int32_t** col_idx, const int32_t** nnzb_dev);

/* Fused evaluate + differentiate + assemble (section 方法: g = sum S^T g_j,
 * H = sum S^T H_j S_j; per-term forward-mode AD in registers, patch-local
 * pre-reduction in shared memory).  Overwrites every element of g and of
 * the first nnzb blocks of H_vals.
 *   x       DEVICE [V][dof] positions
 *   t       HOST struct; its arrays are DEVICE pointers (see mad_terms)
 *   g       DEVICE [V][dof] gradient (out)
 *   H_vals  DEVICE [capacity_blocks][dof][dof] Hessian values (out)
 *   energy  DEVICE double (out) or NULL to skip the energy
 * MAD_TERM_PAIR uses the pair set of the latest mad_add_pairs on this
 * context.  Errors: MAD_ERR_INVALID_ARG (NULL array for an active term,
 * SYMDIR with dof 3), MAD_ERR_CUDA (launch failure).                       */
mad_status mad_eval(mad_ctx* c, const void* x, const mad_terms* t, void* g,
                    void* H_vals, double* energy, void* stream);

/* Matrix-free Hessian-vector product y = H(x) v of the same terms, without
 * forming H (section 实验结果, parameterization with matrix-free HVP).
 *   x, v    DEVICE [V][dof];  y  DEVICE [V][dof] (out, overwritten)     */
mad_status mad_hvp(mad_ctx* c, const void* x, const mad_terms* t,
                   const void* v, void* y, void* stream);

/* Replace the runtime pair set (section 方法, key design 4: interaction
 * discovery is decoupled from evaluation; new off-diagonal blocks are
 * inserted on the GPU into the inactive CSR buffer, which then becomes the
 * active one; no host round trip).
 *   n       number of pairs, 0 <= n <= max_pairs (n = 0 restores the mesh
 *           pattern)
 *   ij      DEVICE [n][2] vertex indices, i != j, any order; duplicates and
 *           pairs on existing mesh edges are allowed and merge into one block
 *   rest    DEVICE [n] rest length r_p of each pair (context dtype)
 * The inputs are read in stream order during the call's kernels; the caller
 * may reuse them once the stream has passed the call.  A pair with an index
 * out of range or i == j is skipped and sets MAD_ERR_INDEX in the device
 * status.  If the merged pattern would exceed capacity_blocks, the device
 * status gets MAD_ERR_CAPACITY and the previous pattern and pair set stay in
 * effect (the new buffer receives a copy of them).
 * Errors returned at once: MAD_ERR_INVALID_ARG, MAD_ERR_CAPACITY
 * (n > max_pairs).                                                         */
mad_status mad_add_pairs(mad_ctx* c, int32_t n, const int32_t* ij,
                         const void* rest, void* stream);

/* Install a set of vertex-face terms (MAD_TERM_VF) on the GPU (section 方法,
 * key design 4: runtime terms are discovered apart from their evaluation,
 * and their new blocks are inserted in parallel on the GPU).
 *   n   number of terms, 0 <= n <= max_pairs / 3
 *   vf  DEVICE [n][2] (vertex p, face f) per term
 * Replaces the pair set with the terms' 3n (p, corner) pairs (as
 * mad_add_pairs would) and builds, on the GPU, the list of the terms that
 * touch each row with their blocks' positions.  mad_eval and mad_hvp with
 * MAD_TERM_VF and t->vf == NULL then evaluate the installed terms: t->vf_n
 * must equal n, t->vf_rest [n] and t->vf_k are read per call.  Each row's
 * thread adds its own share of its terms (gradient and blocks), so the
 * results need no atomics and are reproducible run to run.  A later
 * mad_add_pairs drops the installed set.  A term with an index out of range
 * or a vertex that is a corner of its face is skipped and sets
 * MAD_ERR_INDEX in the device status.  Stream-ordered, no allocation.
 * Errors: MAD_ERR_INVALID_ARG, MAD_ERR_CAPACITY (n > max_pairs / 3),
 * MAD_ERR_UNIMPLEMENTED (dof 2), MAD_ERR_CUDA.                              */
mad_status mad_add_vf(mad_ctx* c, int32_t n, const int32_t* vf, void* stream);

/* ---- vector-valued objective: residuals and sparse Jacobian -------------
 * Section 方法: a vector-valued objective assembles the sparse Jacobian
 * J = sum_j P_j^T J_j S_j (S_j selects a term's stencil, P_j places its
 * residuals in the global residual vector); the highlights note that
 * materialising J explicitly pays off for large geometry problems.
 * Each mesh term contributes a residual vector whose half squared norm is
 * the term's scalar energy, so 1/2 |r|^2 = E, J^T r = g, and J^T J is the
 * Gauss-Newton part of H:
 *   MAD_TERM_SPRING   r = sqrt(k) (|x_a - x_b| - L0)         1 row per edge
 *   MAD_TERM_INERTIA  r = sqrt(w) (x_v - xt_v)              dof rows per vertex
 *   MAD_TERM_SYMDIR   r = sqrt(2A) (vec J, vec J^-1)         8 rows per face
 *                     (vec of a 2x2 matrix: row-major; dof 2 only)
 * Rows are term-major: springs in mad_edges order, then inertia (vertex v,
 * component c at row v*dof + c of that segment), then faces in face order.
 * J is scalar CSR with int64 row pointers and int32 columns; a column is
 * vertex*dof + component, ascending within each row (the stencil's vertices
 * sorted by index).  Nonzeros per row: 2*dof (spring), 1 (inertia), 6 (face).
 * MAD_TERM_PAIR, MAD_TERM_AREA, MAD_TERM_ARAP and MAD_TERM_VF are not part
 * of the vector objective (MAD_ERR_UNIMPLEMENTED).                          */

/* Rows and nonzeros of the Jacobian of the terms in `mask`.  Errors:
 * MAD_ERR_INVALID_ARG (NULL outputs, unknown bits), MAD_ERR_UNIMPLEMENTED
 * (MAD_TERM_PAIR, MAD_TERM_AREA, MAD_TERM_ARAP, or MAD_TERM_SYMDIR with
 * dof 3).                                                                   */
mad_status mad_jacobian_shape(const mad_ctx* c, uint32_t mask, int64_t* nrows, int64_t* nnz);

/* Writes the Jacobian's pattern for `mask`: row_ptr DEVICE int64 [nrows+1],
 * col_idx DEVICE int32 [nnz] (caller-owned, sized by mad_jacobian_shape).
 * The pattern depends only on the mesh and the mask.  Stream-ordered.       */
mad_status mad_jacobian_pattern(mad_ctx* c, uint32_t mask, int64_t* row_ptr, int32_t* col_idx,
                                void* stream);

/* Residuals and Jacobian values at x for the terms in t->mask (t->flags is
 * ignored): r DEVICE [nrows] and J_vals DEVICE [nnz] in the context dtype,
 * in the order of mad_jacobian_pattern; both are overwritten.  The local
 * Jacobians come from first-order forward AD on each term's natural
 * variables.  Stream-ordered, no allocation, no host synchronisation.
 * Errors: as mad_jacobian_shape, plus MAD_ERR_INVALID_ARG for a NULL array
 * of an active term.                                                        */
mad_status mad_jacobian(mad_ctx* c, const void* x, const mad_terms* t, void* r, void* J_vals,
                        void* stream);

/* Stream capture.  mad_eval, mad_hvp, mad_add_pairs, mad_jacobian_pattern
 * and mad_jacobian only enqueue kernels and memsets on `stream`: they
 * neither allocate nor synchronise, so they can be recorded in a CUDA graph
 * and replayed with new data in the captured buffers.  Host-side choices
 * are fixed at capture: the number of pairs passed to mad_add_pairs, the
 * term mask and flags, and which of the two CSR buffers each captured call
 * reads or writes.  mad_status_sync, mad_eval_host, mad_create and
 * mad_destroy synchronise or allocate and cannot be captured.               */

/* Synchronise `stream`, read and clear the sticky device status word and
 * return it (MAD_OK when no device-side error was recorded).  Off the hot
 * path by design.                                                          */
mad_status mad_status_sync(mad_ctx* c, void* stream);

/* mad_eval for callers whose data lives in HOST memory: copies x to the
 * device, evaluates, copies g, H_vals and the energy back, and synchronises
 * `stream` before returning.  x, g, H_vals, energy are HOST pointers (pinned
 * memory gives full copy bandwidth); energy may be NULL.  The term
 * parameter arrays in *t stay DEVICE pointers.  H_vals receives nnzb blocks
 * where nnzb is the current pattern's block count.  The first call
 * allocates the context's device staging buffers for x, g and H_vals.      */
mad_status mad_eval_host(mad_ctx* c, const void* x, const mad_terms* t,
                         void* g, void* H_vals, double* energy, void* stream);

/* Human-readable description of the last error on this context (or of the
 * last failed mad_create when c is NULL).  Never NULL.                     */
const char* mad_last_error(const mad_ctx* c);

/* Release every resource of the context (synchronises the device first).  */
void mad_destroy(mad_ctx* c);

/* Total energy of the given terms, for callers that cannot allocate device
 * memory: code whose device memory is owned by another allocator (a caching
 * allocator of a host framework that has reserved the GPU), and loops that
 * must not allocate after their set-up.  Such callers cannot create a
 * context either (mad_create allocates), so everything is passed in: all
 * arrays are DEVICE pointers in dtype `dt` (index arrays int32), `t` is a
 * HOST struct as for mad_eval, and `energy` is a DEVICE double (out).
 *   springs  nE edges [nE][2] with t->spring_rest [nE] (e.g. mad_edges order)
 *   inertia  the V vertices with t->inertia_xt [V][dof]
 *   faces    nF faces F [nF][3]: with dof 2, MAD_TERM_SYMDIR and/or
 *            MAD_TERM_ARAP read t->face_Minv and t->face_area; with dof 3,
 *            MAD_TERM_AREA reads t->face_area (A0) and t->area_k
 *   pairs    nP pairs [nP][2] with pair_rest [nP] and t->pair_k
 * Only the bits of t->mask select terms; t->flags is ignored.  No paper
 * counterpart: it is the energy reduction of mad_eval without a context.
 * Indices: every vertex index of edges, F and pairs should lie in [0, V).  A
 * term with an index outside it is skipped (nothing is read through that
 * index) and makes the energy NaN, so bad input is visible in the result.
 * Memory: the per-block partial sums live in a fixed device array of this
 * library (65,536 doubles, held by every device that loads the library until
 * the process exits); nothing is allocated or freed.  The array is shared by
 * every call on a device and keeps the last call's values; each call writes
 * every slot it reads, so nothing needs clearing, but calls that overlap on
 * the GPU (different streams at once) race.  Each call on a stream that is
 * not being captured looks up the array's device address
 * (cudaGetSymbolAddress); a call under stream capture reuses the address
 * found by the last such call, so make one call before any capture, and
 * again after a cudaDeviceReset.
 * Errors: MAD_ERR_INVALID_ARG (sizes, dtype, missing arrays, unknown mask
 * bits), MAD_ERR_UNIMPLEMENTED (MAD_TERM_SYMDIR or MAD_TERM_ARAP with dof
 * other than 2, MAD_TERM_AREA with dof other than 3, any MAD_TERM_VF bit),
 * MAD_ERR_CAPACITY (more than 16,777,216 terms in total: the fixed array
 * holds 65,536 sums of 256 terms), MAD_ERR_CUDA.                           */
mad_status mad_energy_noalloc(int32_t V, int32_t dof, mad_dtype dt, const void* x,
                              const mad_terms* t, int32_t nE, const int32_t* edges,
                              int32_t nF, const int32_t* F, int32_t nP,
                              const int32_t* pairs, const void* pair_rest,
                              double* energy, void* stream);

/* ---- owner-computes sharding over several GPUs ---------------------------
 * One mesh split across GPUs by Hessian rows (section 方法, key design 2,
 * carried from patches to GPUs): each GPU owns a contiguous range of rows,
 * evaluates every term that touches an owned vertex, and writes only its
 * rows of g and H, so no reduction is needed; the only exchange is the
 * positions of the vertices across its range's border (its halo), which
 * the evaluation reads directly from their owners' buffers (peer device
 * pointers, e.g. over NVLink).  Each GPU's Hessian values are the contiguous
 * range [block_begin[r], block_begin[r+1]) of the mesh pattern's blocks.  */
#define MAD_MAX_SHARDS 64

/* Split the rows of the mesh pattern of (V, nF, F) into nranks contiguous
 * ranges [row_begin[r], row_begin[r+1]), balanced by block count, every
 * boundary a multiple of 32 rows (or V).  HOST only, no GPU needed.
 *   F            HOST [nF][3] (as for mad_create)
 *   row_begin    HOST int32 [nranks+1] (out); row_begin[0] = 0, [nranks] = V
 *   block_begin  HOST int64 [nranks+1] (out, may be NULL): the mesh
 *                pattern's row_ptr at each boundary
 * Ranges may be empty when V is small.  Errors: MAD_ERR_INVALID_ARG (sizes,
 * 1 <= nranks <= MAD_MAX_SHARDS, a bad face).                              */
mad_status mad_shard_plan(int32_t V, int32_t nF, const int32_t* F, int32_t nranks,
                          int32_t* row_begin, int64_t* block_begin);

/* The halo of rows [row_lo, row_hi): every vertex outside the range that
 * one of its rows couples to (the columns of its mesh-pattern rows outside
 * the range), sorted.  HOST only.  *n_halo receives the count; halo (HOST
 * int32 [cap]) receives the list when cap >= *n_halo (cap = 0 only counts;
 * else MAD_ERR_CAPACITY).  Errors: MAD_ERR_INVALID_ARG.                     */
mad_status mad_shard_halo(int32_t V, int32_t nF, const int32_t* F, int32_t row_lo,
                          int32_t row_hi, int32_t* n_halo, int32_t* halo, int32_t cap);

/* mad_eval for the rows of one shard.  c is a context of the whole mesh
 * (same V and F on every GPU); the mesh pattern must be active (no pair
 * set) and t->mask may hold MAD_TERM_SPRING and MAD_TERM_INERTIA only.
 *   nranks, row_begin  HOST: a plan from mad_shard_plan (or any ranges
 *                      with boundaries at multiples of 32 rows)
 *   x_parts            HOST array of nranks DEVICE pointers: shard s's
 *                      positions [row_begin[s+1] - row_begin[s]][dof] (the
 *                      caller's own part and its peers' parts, readable
 *                      from this device, e.g. peer memory over NVLink)
 *   rank               the shard to evaluate
 *   t                  as for mad_eval, arrays over the whole mesh
 *                      (spring_rest [E], inertia_xt [V][dof])
 *   g_part             DEVICE [rows of the shard][dof] (out)
 *   H_part             DEVICE [block_begin[rank+1] - block_begin[rank]]
 *                      [dof][dof] (out): the shard's blocks of the mesh
 *                      pattern, in order
 *   energy             DEVICE double (out) or NULL: the shard's share of
 *                      the energy (the shares of all shards sum to E)
 * Reads x_parts[s] only at the vertices of shard s in this shard's halo.
 * The caller orders the peers' writes of their parts before this call
 * (e.g. a barrier between steps).  Stream-ordered, no allocation.
 * Errors: MAD_ERR_INVALID_ARG, MAD_ERR_UNIMPLEMENTED (other terms, active
 * pairs, a mesh without compact row tables: see mad_info_t), MAD_ERR_CUDA. */
mad_status mad_eval_shard(mad_ctx* c, int32_t nranks, const int32_t* row_begin,
                          const void* const* x_parts, int32_t rank, const mad_terms* t,
                          void* g_part, void* H_part, double* energy, void* stream);

/* Self-test of the forward-mode number types on the device, used by the test
 * suite.  For each of n inputs (a, b) (HOST double [n][2]) it evaluates, in
 * fp64 hyper-dual arithmetic with tangents seeded on (a, b):
 *   f1 = a sin a,          f2 = a sin b + b cos a,
 *   f3 = sqrt(a^2 + b^2),  f4 = a / b
 * and writes value, gradient (2) and packed Hessian (3) of each: HOST double
 * [n][4][6].  f1 and f2 are the worked examples (Code Examples section) of
 * the page "How to Implement Automatic Differentiation Using the $autodiff
 * Block for Custom Kernels", whose gradients it states in closed form.      */
mad_status mad_selftest_dual(int32_t n, const double* ab, double* out);

#ifdef __cplusplus
}
#endif

#endif /* MAD_H_ */
