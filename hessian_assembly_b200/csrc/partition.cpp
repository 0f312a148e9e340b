// partition.cpp -- host-side patch builder, run once per topology.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法, key design 2: the mesh is cut into small
// patches that fit the GPU memory hierarchy, one CUDA block per patch, with
// ribbon (ghost) elements caching the cross-patch neighbours.  Key design 3:
// the block pattern is preallocated, so each term's destination blocks can be
// looked up once here (the "block-offset lookup") instead of searched per
// evaluation.
//
// Design here (B200 build): patches OWN vertices.  A patch evaluates every
// term that touches one of its owned vertices (terms on the ribbon are thus
// evaluated by every patch that owns one of their vertices) and writes only
// its owned rows.  Patch shapes come from recursive coordinate bisection of
// optional positions (compact, near-square patches), or else from
// breadth-first growth on the vertex graph.  Terms inside a patch are
// greedily coloured so that no two terms of one colour share an owned
// vertex; the kernel accumulates one colour at a time without atomics.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <numeric>
#include <string>
#include <vector>

#include "mad_internal.h"

namespace mad {
namespace {

// Greedy colouring: a term takes the smallest colour not yet used by any of
// its owned vertices.  Colour sets grow as needed (a vertex of valence d
// needs d colours).
struct Colouring {
  std::vector<std::vector<uint64_t>> used;  // per owned local vertex
  explicit Colouring(int no) : used((size_t)no) {}
  int pick(const int* vs, int n) {
    size_t words = 1;
    for (int i = 0; i < n; ++i)
      if (vs[i] >= 0) words = std::max(words, used[vs[i]].size() + 1);
    for (size_t w = 0; w < words; ++w) {
      uint64_t m = 0;
      for (int i = 0; i < n; ++i)
        if (vs[i] >= 0 && w < used[vs[i]].size()) m |= used[vs[i]][w];
      if (~m) {
        const int c = (int)(w * 64) + __builtin_ctzll(~m);
        for (int i = 0; i < n; ++i) {
          if (vs[i] < 0) continue;
          std::vector<uint64_t>& u = used[vs[i]];
          if (u.size() <= w) u.resize(w + 1, 0);
          u[w] |= 1ull << (c & 63);
        }
        return c;
      }
    }
    return -1;
  }
};

inline int find_pos(const int32_t* ci, int32_t b, int32_t e, int32_t col) {
  const int32_t* p = std::lower_bound(ci + b, ci + e, col);
  if (p == ci + e || *p != col) return -1;
  return (int)(p - (ci + b));
}

}  // namespace

std::string build_patches(int V, int nF, const int32_t* F, const int32_t* rp,
                          const int32_t* ci, const double* xyz, int xyz_dim,
                          int target_owned, int max_stage_blocks, HostPatches& out) {
  out = HostPatches();
  if (V == 0) return "";
  if (target_owned < 1) target_owned = 1;
  std::vector<int32_t> len(V), dpos(V);
  std::vector<int64_t> eptr(V + 1, 0);
  for (int v = 0; v < V; ++v) {
    len[v] = rp[v + 1] - rp[v];
    dpos[v] = find_pos(ci, rp[v], rp[v + 1], v);
    if (dpos[v] < 0) return "pattern row without diagonal";
    if (len[v] > 0xFFFE) return "vertex valence too large for 16-bit block positions";
    if (len[v] > max_stage_blocks)
      return "a single Hessian row exceeds the shared-memory staging budget";
    eptr[v + 1] = eptr[v] + (len[v] - dpos[v] - 1);
  }

  // ---- 1. vertex order and patch boundaries ------------------------------
  std::vector<int32_t> order(V);
  std::vector<int32_t> cuts;  // patch p = order[cuts[p] .. cuts[p+1])
  if (xyz != nullptr) {
    std::iota(order.begin(), order.end(), 0);
    struct Range { int b, e; };
    std::vector<Range> stack{{0, V}};
    while (!stack.empty()) {
      Range r = stack.back();
      stack.pop_back();
      int size = r.e - r.b;
      int64_t maxlen = 1;
      double lo[3] = {1e300, 1e300, 1e300}, hi[3] = {-1e300, -1e300, -1e300};
      for (int i = r.b; i < r.e; ++i) {
        int v = order[i];
        maxlen = std::max<int64_t>(maxlen, len[v]);
        for (int a = 0; a < xyz_dim; ++a) {
          lo[a] = std::min(lo[a], xyz[(size_t)v * xyz_dim + a]);
          hi[a] = std::max(hi[a], xyz[(size_t)v * xyz_dim + a]);
        }
      }
      // rows are staged at a fixed stride (the longest row of the patch)
      const int64_t blocks = (int64_t)size * maxlen;
      if (size <= target_owned && blocks <= max_stage_blocks) {
        cuts.push_back(r.b);
        continue;
      }
      int64_t k1 = (size + target_owned - 1) / target_owned;
      int64_t k2 = (blocks + max_stage_blocks - 1) / max_stage_blocks;
      int64_t k = std::max<int64_t>(2, std::max(k1, k2));
      int64_t kl = k / 2;
      int m = r.b + (int)std::llround((double)size * (double)kl / (double)k);
      m = std::min(std::max(m, r.b + 1), r.e - 1);
      int axis = 0;
      for (int a = 1; a < xyz_dim; ++a)
        if (hi[a] - lo[a] > hi[axis] - lo[axis]) axis = a;
      auto less = [&](int32_t u, int32_t w) {
        double cu = xyz[(size_t)u * xyz_dim + axis], cw = xyz[(size_t)w * xyz_dim + axis];
        return cu < cw || (cu == cw && u < w);
      };
      std::nth_element(order.begin() + r.b, order.begin() + m, order.begin() + r.e, less);
      stack.push_back({m, r.e});
      stack.push_back({r.b, m});
    }
    cuts.push_back(V);
    // the DFS visits leaves left to right; cuts were pushed in that order
  } else {
    std::vector<char> taken(V, 0);
    std::vector<int32_t> seeds, queue;
    size_t seed_head = 0;
    int next_unassigned = 0, pos = 0;
    while (pos < V) {
      int seed = -1;
      while (seed_head < seeds.size() && seed < 0) {
        int c = seeds[seed_head++];
        if (!taken[c]) seed = c;
      }
      if (seed < 0) {
        while (taken[next_unassigned]) ++next_unassigned;
        seed = next_unassigned;
      }
      cuts.push_back(pos);
      queue.clear();
      queue.push_back(seed);
      taken[seed] = 1;
      size_t qh = 0;
      int64_t maxlen = 1;
      int cnt = 0;
      while (qh < queue.size()) {
        int v = queue[qh++];
        const int64_t ml = std::max<int64_t>(maxlen, len[v]);
        if (cnt >= target_owned || (cnt + 1) * ml > max_stage_blocks) {
          taken[v] = 0;  // give it back; it seeds a later patch
          seeds.push_back(v);
          continue;
        }
        order[pos++] = v;
        ++cnt;
        maxlen = ml;
        for (int q = rp[v]; q < rp[v + 1]; ++q) {
          int b = ci[q];
          if (!taken[b]) {
            taken[b] = 1;
            queue.push_back(b);
          }
        }
      }
    }
    cuts.push_back(V);
  }
  const int P = (int)cuts.size() - 1;

  // ---- 2. vertex -> face incidence ------------------------------------------
  std::vector<int32_t> vf_ptr(V + 1, 0), vf(3 * (size_t)nF);
  for (int64_t c = 0; c < 3 * (int64_t)nF; ++c) vf_ptr[F[c] + 1]++;
  for (int v = 0; v < V; ++v) vf_ptr[v + 1] += vf_ptr[v];
  {
    std::vector<int32_t> cur(vf_ptr.begin(), vf_ptr.end() - 1);
    for (int64_t c = 0; c < 3 * (int64_t)nF; ++c) vf[cur[F[c]]++] = (int32_t)(c / 3);
  }

  // ---- 3. per-patch tables ---------------------------------------------------
  std::vector<int32_t> owner(V, -1), lidx(V, -1), stamp(V, -1);
  for (int p = 0; p < P; ++p)
    for (int i = cuts[p]; i < cuts[p + 1]; ++i) owner[order[i]] = p;

  struct ETerm { EdgeLut l; int32_t eid; int colour; };
  struct FTerm { FaceLut l; int colour; };
  std::vector<ETerm> et;
  std::vector<FTerm> ft;
  std::vector<int32_t> owned, halo;
  for (int p = 0; p < P; ++p) {
    owned.assign(order.begin() + cuts[p], order.begin() + cuts[p + 1]);
    std::sort(owned.begin(), owned.end());
    const int no = (int)owned.size();
    halo.clear();
    for (int r = 0; r < no; ++r) {
      int a = owned[r];
      lidx[a] = r;
      stamp[a] = p;
    }
    for (int r = 0; r < no; ++r) {
      int a = owned[r];
      for (int q = rp[a]; q < rp[a + 1]; ++q) {
        int b = ci[q];
        if (stamp[b] != p) {
          stamp[b] = p;
          halo.push_back(b);
        }
      }
    }
    std::sort(halo.begin(), halo.end());
    const int nv = no + (int)halo.size();
    if (nv > 0xFFFE) return "patch has too many vertices for 16-bit local indices";
    for (size_t h = 0; h < halo.size(); ++h) lidx[halo[h]] = no + (int)h;

    PatchHdr H;
    std::memset(&H, 0, sizeof(H));
    // per-patch arrays start on 16-byte boundaries so the kernel can copy
    // them to shared memory in 16-byte pieces
    while (out.vgid.size() % 4 != 0) {
      out.vgid.push_back(0);
      out.meta.push_back(make_uint2(0, 0));
    }
    H.vbeg = (int)out.vgid.size();
    H.nv = nv;
    H.no = no;
    int nstage = 0, stride = 1;
    for (int r = 0; r < no; ++r) {
      nstage += len[owned[r]];
      stride = std::max(stride, (int)len[owned[r]]);
    }
    H.nstage = nstage;
    H.stride = stride;
    // runs of consecutive vertex ids
    H.rbeg = (int)out.runs.size();
    std::vector<int> run_of(no), run_start(no);
    for (int r = 0; r < no; ++r) {
      if (r == 0 || owned[r] != owned[r - 1] + 1) {
        out.runs.push_back((uint32_t)r);
        run_start[r] = r;
      } else {
        run_start[r] = run_start[r - 1];
      }
      run_of[r] = (int)out.runs.size() - 1 - H.rbeg;
      out.runs.back() += 1u << 16;  // one more row in this run
    }
    H.nruns = (int)out.runs.size() - H.rbeg;
    for (int r = 0; r < no; ++r) {
      out.vgid.push_back(owned[r]);
      uint2 m;
      m.x = pack_meta(len[owned[r]], dpos[owned[r]]);
      m.y = (uint32_t)run_start[r] | ((uint32_t)run_of[r] << 16);
      out.meta.push_back(m);
    }
    for (int h : halo) {
      out.vgid.push_back(h);
      out.meta.push_back(make_uint2(0, 0));
    }
    // row slots: column local index + edge id for every mesh-pattern block,
    // each row padded to the stride
    while (out.slot_lidx.size() % 8 != 0) {
      out.slot_lidx.push_back(kNoSlot);
      out.slot_eid.push_back(-1);
    }
    H.sbeg = (int)out.slot_lidx.size();
    for (int r = 0; r < no; ++r) {
      const int a = owned[r];
      for (int q = rp[a]; q < rp[a] + stride; ++q) {
        if (q >= rp[a + 1]) {
          out.slot_lidx.push_back(kNoSlot);
          out.slot_eid.push_back(-1);
          continue;
        }
        const int b = ci[q];
        out.slot_lidx.push_back((uint16_t)lidx[b]);
        if (b == a) {
          out.slot_eid.push_back(-1);
        } else if (a < b) {
          out.slot_eid.push_back((int32_t)(eptr[a] + (q - rp[a]) - dpos[a] - 1));
        } else {
          const int pba = find_pos(ci, rp[b], rp[b + 1], a);
          out.slot_eid.push_back((int32_t)(eptr[b] + pba - dpos[b] - 1));
        }
      }
    }

    // edge terms: every edge with at least one owned endpoint, once
    et.clear();
    Colouring ce(no);
    for (int r = 0; r < no; ++r) {
      int a = owned[r];
      for (int q = rp[a]; q < rp[a + 1]; ++q) {
        int b = ci[q];
        if (b == a) continue;
        bool b_owned = owner[b] == p;
        if (b_owned && b < a) continue;
        ETerm t;
        t.l.la = (uint16_t)r;
        t.l.lb = (uint16_t)lidx[b];
        t.l.pab = (uint16_t)(q - rp[a]);
        int pba = find_pos(ci, rp[b], rp[b + 1], a);
        if (pba < 0) return "pattern is not symmetric";
        t.l.pba = b_owned ? (uint16_t)pba : kNotOwned;
        if (a < b)
          t.eid = (int32_t)(eptr[a] + (q - rp[a]) - dpos[a] - 1);
        else
          t.eid = (int32_t)(eptr[b] + pba - dpos[b] - 1);
        int vs[2] = {r, b_owned ? lidx[b] : -1};
        t.colour = ce.pick(vs, 2);
        et.push_back(t);
      }
    }
    std::stable_sort(et.begin(), et.end(), [](const ETerm& u, const ETerm& w) {
      return u.colour != w.colour ? u.colour < w.colour : u.eid < w.eid;
    });
    H.ebeg = (int)out.elut.size();
    H.ne = (int)et.size();
    H.ecbeg = (int)out.ecol.size();
    int nce = et.empty() ? 0 : et.back().colour + 1;
    H.nce = nce;
    {
      size_t i = 0;
      for (int c = 0; c <= nce; ++c) {
        while (i < et.size() && et[i].colour < c) ++i;
        out.ecol.push_back((int32_t)i);
      }
    }
    for (const ETerm& t : et) {
      out.elut.push_back(t.l);
      out.eid.push_back(t.eid);
    }

    // face terms: every face with at least one owned corner, once
    ft.clear();
    if (nF > 0) {
      Colouring cf(no);
      for (int r = 0; r < no; ++r) {
        int a = owned[r];
        for (int k = vf_ptr[a]; k < vf_ptr[a + 1]; ++k) {
          int f = vf[k];
          const int32_t* c = F + 3 * (size_t)f;
          int first = -1;
          for (int m = 0; m < 3; ++m)
            if (owner[c[m]] == p && (first < 0 || c[m] < first)) first = c[m];
          if (first != a) continue;
          FTerm t;
          int vs[3];
          for (int kk = 0; kk < 3; ++kk) {
            t.l.l[kk] = (uint16_t)lidx[c[kk]];
            bool own = owner[c[kk]] == p;
            vs[kk] = own ? lidx[c[kk]] : -1;
            for (int m = 0; m < 3; ++m) {
              if (!own) {
                t.l.pos[kk][m] = kNotOwned;
                continue;
              }
              int ps = find_pos(ci, rp[c[kk]], rp[c[kk] + 1], c[m]);
              if (ps < 0) return "face corner missing from pattern";
              t.l.pos[kk][m] = (uint16_t)ps;
            }
          }
          t.l.fid = f;
          t.colour = cf.pick(vs, 3);
          ft.push_back(t);
        }
      }
      std::stable_sort(ft.begin(), ft.end(), [](const FTerm& u, const FTerm& w) {
        return u.colour != w.colour ? u.colour < w.colour : u.l.fid < w.l.fid;
      });
    }
    H.fbeg = (int)out.flut.size();
    H.nf = (int)ft.size();
    H.fcbeg = (int)out.fcol.size();
    int ncf = ft.empty() ? 0 : ft.back().colour + 1;
    H.ncf = ncf;
    {
      size_t i = 0;
      for (int c = 0; c <= ncf; ++c) {
        while (i < ft.size() && ft[i].colour < c) ++i;
        out.fcol.push_back((int32_t)i);
      }
    }
    for (const FTerm& t : ft) out.flut.push_back(t.l);

    out.hdr.push_back(H);
    out.nv_max = std::max(out.nv_max, nv);
    out.no_max = std::max(out.no_max, no);
    out.slots_max = std::max(out.slots_max, no * H.stride);
  }
  // slack so that 16-byte copies rounded up past a patch's end stay in bounds
  for (int i = 0; i < 8; ++i) {
    out.vgid.push_back(0);
    out.meta.push_back(make_uint2(0, 0));
    out.slot_lidx.push_back(kNoSlot);
    out.slot_eid.push_back(-1);
  }
  return "";
}

std::string build_row_tables(int V, const int32_t* rp, const int32_t* ci, int s0_cap,
                             HostRowTables& out) {
  out = HostRowTables();
  std::vector<int32_t> dpos(V);
  std::vector<int64_t> eptr(V + 1, 0);
  int maxoff = 0;
  for (int v = 0; v < V; ++v) {
    dpos[v] = find_pos(ci, rp[v], rp[v + 1], v);
    if (dpos[v] < 0) return "pattern row without diagonal";
    const int len = rp[v + 1] - rp[v];
    if (len > 0xFFFF) return "vertex valence too large";
    maxoff = std::max(maxoff, len - 1);
    eptr[v + 1] = eptr[v] + (len - dpos[v] - 1);
  }
  const int s0 = std::max(1, std::min(maxoff, s0_cap));
  out.s0 = s0;
  const int ntiles = (V + 31) / 32;
  out.slots.assign((size_t)ntiles * s0 * 32, make_int2(-1, -1));
  out.meta.resize(V);
  out.ofl_ptr.assign(V + 1, 0);
  for (int v = 0; v < V; ++v) {
    const int len = rp[v + 1] - rp[v];
    out.meta[v] = (uint32_t)(len - 1) | ((uint32_t)dpos[v] << 16);
    out.ofl_ptr[v + 1] = out.ofl_ptr[v] + std::max(0, len - 1 - s0);
  }
  out.ofl.resize(std::max<int32_t>(1, out.ofl_ptr[V]));
  for (int v = 0; v < V; ++v) {
    int k = 0;
    const int t = v / 32, l = v % 32;
    for (int q = rp[v]; q < rp[v + 1]; ++q) {
      const int b = ci[q];
      if (b == v) continue;
      int32_t eid;
      if (v < b) {
        eid = (int32_t)(eptr[v] + (q - rp[v]) - dpos[v] - 1);
      } else {
        const int pba = find_pos(ci, rp[b], rp[b + 1], v);
        eid = (int32_t)(eptr[b] + pba - dpos[b] - 1);
      }
      const int2 e = make_int2(b, eid);
      if (k < s0)
        out.slots[((size_t)t * s0 + k) * 32 + l] = e;
      else
        out.ofl[out.ofl_ptr[v] + (k - s0)] = e;
      ++k;
    }
  }
  // the compact slots, when every delta fits its 16 bits
  out.ctile.resize(ntiles);
  out.cslots.assign((size_t)ntiles * s0 * 32, 0u);
  bool fits = true;
  for (int t = 0; t < ntiles && fits; ++t) {
    const int v0 = 32 * t;
    uint32_t ofl_mask = 0;
    for (int l = 0; l < 32 && v0 + l < V; ++l)
      if (out.ofl_ptr[v0 + l + 1] > out.ofl_ptr[v0 + l]) ofl_mask |= 1u << l;
    out.ctile[t] = make_int4(rp[v0], (int32_t)eptr[v0], (int32_t)ofl_mask, 0);
    for (int k = 0; k < s0 && fits; ++k)
      for (int l = 0; l < 32; ++l) {
        const size_t q = ((size_t)t * s0 + k) * 32 + l;
        const int2 e = out.slots[q];
        if (e.x < 0) continue;
        const int64_t dc = (int64_t)e.x - (v0 + l), de = (int64_t)e.y - eptr[v0];
        if (dc < -32768 || dc > 32767 || de < -32768 || de > 32767) {
          fits = false;
          break;
        }
        out.cslots[q] = (uint32_t)(uint16_t)(int16_t)dc | ((uint32_t)(uint16_t)(int16_t)de << 16);
      }
  }
  if (!fits) {
    out.ctile.clear();
    out.cslots.clear();
  }
  return "";
}

std::string build_face_rows(int V, int nF, const int32_t* F, const int32_t* rp,
                            const int32_t* ci, HostFaceRows& out) {
  out = HostFaceRows();
  if ((int64_t)nF * 3 >= (int64_t)0x7FFFFFFF) return "too many faces for 3f + c";
  for (int v = 0; v < V; ++v)
    if (rp[v + 1] - rp[v] >= (1 << kFacePosBits)) return "row too long for face positions";
  std::vector<int32_t> cnt(V + 1, 0);
  for (int64_t f = 0; f < nF; ++f)
    for (int c = 0; c < 3; ++c) ++cnt[F[3 * f + c] + 1];
  int maxdeg = 0;
  for (int v = 0; v < V; ++v) maxdeg = std::max(maxdeg, cnt[v + 1]);
  const int sf = std::max(1, std::min(maxdeg, kFaceRowSlots));
  out.sf = sf;
  const int ntiles = (V + 31) / 32;
  out.slots.assign((size_t)ntiles * sf * 32, make_int4(-1, -1, -1, 0));
  out.ofl_ptr.assign(V + 1, 0);
  for (int v = 0; v < V; ++v) out.ofl_ptr[v + 1] = out.ofl_ptr[v] + std::max(0, cnt[v + 1] - sf);
  out.ofl.resize(std::max<int32_t>(1, out.ofl_ptr[V]));
  out.cslots.assign((size_t)ntiles * sf * 32, -1);
  out.cofl.resize(out.ofl.size());
  std::vector<int32_t> fill(V, 0);
  for (int64_t f = 0; f < nF; ++f) {  // face order within each row
    for (int c = 0; c < 3; ++c) {
      const int i = F[3 * f + c], j = F[3 * f + (c + 1) % 3], k = F[3 * f + (c + 2) % 3];
      const int pj = find_pos(ci, rp[i], rp[i + 1], j);
      const int pk = find_pos(ci, rp[i], rp[i + 1], k);
      if (pj < 0 || pk < 0) return "face edge missing from the pattern";
      const uint32_t w = (uint32_t)c | ((uint32_t)pj << 2) | ((uint32_t)pk << (2 + kFacePosBits));
      const int s = fill[i]++;
      // the last slot of a row that continues in the overflow table carries
      // the sign bit of k
      const bool more = s == sf - 1 && cnt[i + 1] > sf;
      const int4 e = make_int4((int32_t)f, j, more ? (int32_t)((uint32_t)k | 0x80000000u) : k,
                               (int32_t)w);
      const int32_t fc = (int32_t)(3 * f + c);
      if (s < sf) {
        out.slots[((size_t)(i / 32) * sf + s) * 32 + i % 32] = e;
        out.cslots[((size_t)(i / 32) * sf + s) * 32 + i % 32] =
            more ? (int32_t)((uint32_t)fc | 0x80000000u) : fc;
      } else {
        out.ofl[out.ofl_ptr[i] + (s - sf)] = e;
        out.cofl[out.ofl_ptr[i] + (s - sf)] = fc;
      }
    }
  }
  return "";
}

}  // namespace mad
