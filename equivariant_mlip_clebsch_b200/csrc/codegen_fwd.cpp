// codegen_fwd.cpp -- the forward CGTP convolution kernel, generated per plan.
//
// Execution (node-centric, as in LunaTP Fig. 3a: every receiver's row is
// accumulated on chip and stored once, no atomics):
//   grid (n_recv, S): CTA (i, s) owns receiver i and slice s of the warp roles.
//   warp NW (producer): streams the receiver's edges in chunks of B through a
//     ring of STAGES shared-memory stages -- W rows and x rows by bulk copy
//     (cp.async.bulk, completion counted on an mbarrier), Y rows by plain
//     loads -- and waits for each stage to be released before refilling it.
//   warps 0..NW-1 (consumers): per chunk, build
//       Chat_{e,p}[m3][m1] = sum_m2 C_p[m1][m2][m3] Y[e][l2^2+m2]
//     for every path of the slice (shared by all channels), then each warp
//     runs its role: R channels per lane of one hidden irrep and a group of
//     that irrep's paths, accumulating
//       acc[p][u][m3] += W[e][k0_p+u] * sum_m1 Chat[m3][m1] x[j][u][m1]
//     in registers.  The role code is specialised to its degrees and offsets.
// The paths of a hidden irrep are grouped under a register budget per lane
// (the output-component budget idea of LunaTP Fig. 3b / Table 7); x is
// loaded once per edge for all paths of a group (Table 8's cross-path reuse).
#include <algorithm>
#include <array>
#include <cstdio>
#include <cstdlib>
#include <cmath>
#include <cstring>
#include <map>
#include <numeric>
#include <sstream>

#include "codegen_common.hpp"

namespace cgtp {

// Producer warp: streams chunks of the receiver's edges into the stage ring.
// Shared by the forward and backward generators.
std::string gen_producer(const Plan& P, const FwdConfig& F) {
  std::ostringstream o;
  o << "__device__ __noinline__ void producer(const int* __restrict__ col, const float* __restrict__ x,\n"
       "    const float* __restrict__ Y, const float* __restrict__ W, int* __restrict__ err,\n"
       "    unsigned char* smem, int slice, int e0, int e1, int lane) {\n"
       "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
       "  const int nchunk = (e1 - e0 + NB - 1) / NB;\n"
       "  const u64 pol = policy_evict_first();\n"
       "  (void)pol;\n"
       "  bool dead = false;\n"
       "  for (int c = 0; c < nchunk; ++c) {\n"
       "    const int s = c % NSTAGE;\n"
       "    if (c >= NSTAGE && !mbar_wait(empty0 + 8 * s, ((c / NSTAGE) - 1) & 1)) { dead = true; break; }\n"
       "    const int eb = e0 + c * NB;\n"
       "    const int nb = min(NB, e1 - eb);\n"
       "    unsigned char* st = smem + OFF_STAGE + s * STAGE_BYTES;\n"
       "    float* sY = reinterpret_cast<float*>(st + W_BYTES + X_BYTES);\n"
       "    for (int t = lane; t < nb * DE; t += 32) sY[t] = Y[(size_t)eb * DE + t];\n";
  if (F.x_smem) o << "    const int jj = (lane < nb) ? col[eb + lane] : 0;\n";
  o << "    if (lane == 0) {\n      u32 tx = 0;\n";
  if (F.w_smem) o << "      tx += (u32)nb * NU * 4;\n";
  if (F.x_smem) o << "      tx += (u32)nb * slice_xbytes(slice);\n";
  o << "      mbar_expect_tx(full0 + 8 * s, tx);\n    }\n    __syncwarp();\n";
  if (F.w_smem)
    o << "    if (lane == 0) bulk_g2s_stream(smem_u32(st), W + (size_t)eb * NU, (u32)nb * NU * 4, full0 + 8 * s, pol);\n";
  if (F.x_smem)
    o << "    if (lane < nb) stage_x(slice, smem_u32(st + W_BYTES) + lane * XS * 4, x + (size_t)jj * DIN, full0 + 8 * s);\n";
  o << "    mbar_arrive(full0 + 8 * s);  // releases this lane's Y stores\n"
       "  }\n"
       "  if (dead && lane == 0) atomicOr(err, 10);\n"
       "  // copies still in flight must land before the CTA may exit\n"
       "  if (lane == 0)\n"
       "    for (int c = max(0, nchunk - NSTAGE); c < nchunk; ++c) mbar_wait(full0 + 8 * (c % NSTAGE), (c / NSTAGE) & 1);\n"
       "}\n";
  // Chat build of one chunk by all consumer threads
  o << "__device__ __forceinline__ void chat_build(const int4* __restrict__ sent, int nent,\n"
       "    const int2* __restrict__ term, const float* __restrict__ sY, float* __restrict__ ch, int chs,\n"
       "    int nb, int tid) {\n"
       "  for (int t = tid; t < nb * nent; t += NW * 32) {\n"
       "    const int b = t / nent, q = t - b * nent;\n"
       "    const int4 en = sent[q];\n"
       "    float v = 0.f;\n"
       "    for (int k = 0; k < en.z; ++k) {\n"
       "      const int2 tm = term[en.y + k];\n"
       "      v = fmaf(__int_as_float(tm.y), sY[b * DE + tm.x], v);\n"
       "    }\n"
       "    ch[b * chs + en.x] = v;\n"
       "  }\n"
       "}\n";
  return o.str();
}

// Per-slice helpers: Chat size, x staging (bulk copies of the slice's hidden
// irrep blocks) and its byte count.
std::string gen_slice_helpers(const Plan& P, const FwdConfig& F, const std::vector<SliceLayout>& SL) {
  std::ostringstream o;
  const int S = F.S;
  o << "__device__ __forceinline__ int slice_chs(int s) { switch (s) {";
  for (int s = 0; s < S; ++s) o << " case " << s << ": return " << SL[s].chs << ";";
  o << " } return 0; }\n";
  if (F.x_smem) {
    o << "__device__ __forceinline__ void stage_x(int s, u32 dst, const float* xrow, u32 bar) {\n  switch (s) {\n";
    for (int s = 0; s < S; ++s) {
      o << "  case " << s << ":\n";
      std::vector<std::array<int, 3>> cp;
      for (int a : SL[s].irreps) {
        const int src = P.x_off[a], dst = SL[s].x_st.at(a), n = P.in[a].mul * (2 * P.in[a].l + 1);
        if (!cp.empty() && cp.back()[0] + cp.back()[2] == src && cp.back()[1] + cp.back()[2] == dst)
          cp.back()[2] += n;
        else
          cp.push_back({src, dst, n});
      }
      for (auto& c : cp)
        o << "    bulk_g2s(dst + " << c[1] * 4 << ", xrow + " << c[0] << ", " << c[2] * 4 << ", bar);\n";
      o << "    break;\n";
    }
    o << "  }\n}\n";
    o << "__device__ __forceinline__ u32 slice_xbytes(int s) { switch (s) {";
    for (int s = 0; s < S; ++s) {
      int n = 0;
      for (int a : SL[s].irreps) n += P.in[a].mul * (2 * P.in[a].l + 1);
      o << " case " << s << ": return " << n * 4 << ";";
    }
    o << " } return 0; }\n";
  }
  return o.str();
}

// Shared-memory layout common to both kernels; returns the #defines.
std::string gen_layout(const Plan& P, const FwdConfig& F, const std::vector<SliceLayout>& SL,
                       int extra_bytes, int& off_extra, int& smem_bytes) {
  int XS = 0, CHS = 0;
  for (const auto& sl : SL) {
    XS = std::max(XS, sl.xs);
    CHS = std::max(CHS, sl.chs);
  }
  auto r128 = [](int v) { return (v + 127) & ~127; };
  const int B = F.B, ST = F.stages;
  const int bar_bytes = r128(2 * ST * 8);
  const int w_bytes = F.w_smem ? r128(B * (int)P.U * 4) : 0;
  const int x_bytes = F.x_smem ? r128(B * XS * 4) : 0;
  const int y_bytes = r128(B * (int)P.D_e * 4);
  const int stage_bytes = w_bytes + x_bytes + y_bytes;
  const int off_stage = bar_bytes;
  const int off_ch = off_stage + ST * stage_bytes;
  off_extra = off_ch + r128(2 * B * CHS * 4);
  smem_bytes = off_extra + r128(extra_bytes);
  std::ostringstream o;
  o << "#define NW " << F.nw << "\n#define NB " << B << "\n#define NSTAGE " << ST
    << "\n#define DIN " << P.D_in << "\n#define DE " << P.D_e << "\n#define DOUT " << P.D_out
    << "\n#define NU " << P.U << "\n#define CHS " << CHS << "\n#define XS " << XS
    << "\n#define STAGE_BYTES " << stage_bytes << "\n#define OFF_STAGE " << off_stage
    << "\n#define OFF_CH " << off_ch << "\n#define W_BYTES " << w_bytes << "\n#define X_BYTES "
    << x_bytes << "\n";
  o << "#define LDW(p) " << (F.w_smem ? "(*(p))" : "ld_stream(p)") << "\n";
  o << "#define LDX(p) " << (F.x_smem ? "(*(p))" : "__ldg(p)") << "\n";
  return o.str();
}

static std::string gen_fwd_source(const Plan& P, const std::vector<SliceLayout>& SL,
                                  const std::string& kname, int& smem_bytes) {
  const FwdConfig& F = P.fcfg;
  const int S = F.S, NW = F.nw;
  int off_extra = 0;
  std::ostringstream o;
  o << kPrelude;
  o << gen_layout(P, F, SL, 0, off_extra, smem_bytes);
  o << gen_slice_helpers(P, F, SL);
  o << gen_producer(P, F);

  // role shapes: (irrep, R, path group) with the channel block as a runtime
  // argument; one noinline consumer function per shape and slice layout
  std::vector<int> shape_of(P.fwd_roles.size(), -1);
  std::vector<int> shape_rep;  // representative role of each shape
  std::vector<int> slice_of(P.fwd_roles.size(), -1);
  for (int s = 0; s < S; ++s)
    for (int v : F.slice_roles[s]) slice_of[v] = s;
  for (size_t ri = 0; ri < P.fwd_roles.size(); ++ri) {
    const FwdRole& r = P.fwd_roles[ri];
    for (size_t k = 0; k < shape_rep.size(); ++k) {
      const FwdRole& q = P.fwd_roles[shape_rep[k]];
      if (q.irrep == r.irrep && q.R == r.R && q.paths == r.paths && slice_of[shape_rep[k]] == slice_of[ri]) {
        shape_of[ri] = (int)k;
        break;
      }
    }
    if (shape_of[ri] < 0) {
      shape_of[ri] = (int)shape_rep.size();
      shape_rep.push_back((int)ri);
    }
  }
  for (size_t k = 0; k < shape_rep.size(); ++k) {
    const FwdRole& r = P.fwd_roles[shape_rep[k]];
    const SliceLayout& sl = SL[slice_of[shape_rep[k]]];
    const Irrep& h = P.in[r.irrep];
    const int N1 = 2 * h.l + 1, R = r.R, MUL = h.mul;
    int nacc = 0;
    for (int pi : r.paths) nacc += R * (2 * P.paths[pi].l3 + 1);
    const int xoff = F.x_smem ? sl.x_st.at(r.irrep) : P.x_off[r.irrep];
    o << "// shape " << k << ": irrep " << r.irrep << " (" << h.mul << "x" << h.l << "), " << r.paths.size()
      << " paths, R=" << R << "\n";
    o << "__device__ __noinline__ void fcons_" << k
      << "(const int* __restrict__ col, const float* __restrict__ x, const float* __restrict__ W,\n"
         "    float* __restrict__ out, const int4* __restrict__ sent, int nent, const int2* __restrict__ term,\n"
         "    int* __restrict__ err, unsigned char* smem, int i, int e0, int e1, int u0, int chs) {\n"
         "  const int lane = threadIdx.x & 31;\n"
         "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
         "  const int nchunk = (e1 - e0 + NB - 1) / NB;\n"
         "  float acc[" << nacc << "];\n"
         "#pragma unroll\n  for (int k = 0; k < " << nacc << "; ++k) acc[k] = 0.f;\n"
         "  bool ok[" << R << "];\n"
         "#pragma unroll\n  for (int r = 0; r < " << R << "; ++r) ok[r] = u0 + r * 32 + lane < " << MUL << ";\n"
         "  bool dead = false;\n"
         "  for (int c = 0; c < nchunk; ++c) {\n"
         "    const int s = c % NSTAGE;\n"
         "    if (!dead && !mbar_wait(full0 + 8 * s, (c / NSTAGE) & 1)) { dead = true; if (lane == 0) atomicOr(err, 10); }\n"
         "    const int eb = e0 + c * NB;\n"
         "    const int nb = min(NB, e1 - eb);\n"
         "    unsigned char* st = smem + OFF_STAGE + s * STAGE_BYTES;\n"
         "    const float* sY = reinterpret_cast<const float*>(st + W_BYTES + X_BYTES);\n"
         "    float* ch = reinterpret_cast<float*>(smem + OFF_CH) + (c & 1) * NB * CHS;\n"
         "    if (!dead) chat_build(sent, nent, term, sY, ch, chs, nb, threadIdx.x);\n"
         "    consumer_bar(NW * 32);\n"
         "    if (!dead) {\n"
         "      for (int b = 0; b < nb; ++b) {\n"
         "        const float* chb = ch + b * chs;\n";
    if (F.w_smem)
      o << "        const float* wr = reinterpret_cast<const float*>(st) + b * NU;\n";
    else
      o << "        const float* wr = W + (size_t)(eb + b) * NU;\n";
    if (F.x_smem)
      o << "        const float* xr = reinterpret_cast<const float*>(st + W_BYTES) + b * XS + " << xoff << ";\n";
    else
      o << "        const float* xr = x + (size_t)col[eb + b] * DIN + " << xoff << ";\n";
    o << "        float xv[" << R << "][" << N1 << "];\n"
      << "#pragma unroll\n        for (int r = 0; r < " << R << "; ++r) {\n"
      << "          const int u = u0 + r * 32 + lane;\n"
      << "#pragma unroll\n          for (int m1 = 0; m1 < " << N1 << "; ++m1) xv[r][m1] = ok[r] ? LDX(xr + u * "
      << N1 << " + m1) : 0.f;\n        }\n";
    int A = 0;
    for (int pi : r.paths) {
      const Path& p = P.paths[pi];
      const int N3 = 2 * p.l3 + 1;
      o << "        { float w[" << R << "];\n#pragma unroll\n          for (int r = 0; r < " << R
        << "; ++r) w[r] = ok[r] ? LDW(wr + " << p.k0 << " + u0 + r * 32 + lane) : 0.f;\n"
        << "          fpath<" << N1 << "," << N3 << "," << R << "," << A << "," << nacc << ">(acc, chb + "
        << sl.ch_off.at(pi) << ", xv, w); }\n";
      A += R * N3;
    }
    o << "      }\n    }\n    __syncwarp();\n    if (lane == 0) mbar_arrive(empty0 + 8 * s);\n  }\n";
    o << "  float* orow = out + (size_t)i * DOUT;\n";
    A = 0;
    for (int pi : r.paths) {
      const Path& p = P.paths[pi];
      const int N3 = 2 * p.l3 + 1;
      o << "#pragma unroll\n  for (int r = 0; r < " << R << "; ++r) if (ok[r]) {\n    const int u = u0 + r * 32 + lane;\n"
        << "#pragma unroll\n    for (int m3 = 0; m3 < " << N3 << "; ++m3) orow[" << p.o_off << " + u * " << N3
        << " + m3] = acc[" << A << " + r * " << N3 << " + m3];\n  }\n";
      A += R * N3;
    }
    o << "}\n";
  }
  // idle consumer: keeps the barrier and stage accounting of the CTA
  o << "__device__ __noinline__ void fcons_idle(const int4* __restrict__ sent, int nent,\n"
       "    const int2* __restrict__ term, int* __restrict__ err, unsigned char* smem, int e0, int e1, int chs) {\n"
       "  const int lane = threadIdx.x & 31;\n"
       "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
       "  const int nchunk = (e1 - e0 + NB - 1) / NB;\n"
       "  bool dead = false;\n"
       "  for (int c = 0; c < nchunk; ++c) {\n"
       "    const int s = c % NSTAGE;\n"
       "    if (!dead && !mbar_wait(full0 + 8 * s, (c / NSTAGE) & 1)) { dead = true; if (lane == 0) atomicOr(err, 10); }\n"
       "    const int nb = min(NB, e1 - (e0 + c * NB));\n"
       "    unsigned char* st = smem + OFF_STAGE + s * STAGE_BYTES;\n"
       "    const float* sY = reinterpret_cast<const float*>(st + W_BYTES + X_BYTES);\n"
       "    float* ch = reinterpret_cast<float*>(smem + OFF_CH) + (c & 1) * NB * CHS;\n"
       "    if (!dead) chat_build(sent, nent, term, sY, ch, chs, nb, threadIdx.x);\n"
       "    consumer_bar(NW * 32);\n"
       "    __syncwarp();\n"
       "    if (lane == 0) mbar_arrive(empty0 + 8 * s);\n"
       "  }\n"
       "}\n";
  o << "__device__ const int kShape[" << S * NW << "] = {";
  for (int s = 0; s < S; ++s)
    for (int w = 0; w < NW; ++w)
      o << (w < (int)F.slice_roles[s].size() ? shape_of[F.slice_roles[s][w]] : -1) << ",";
  o << "};\n__device__ const int kU0[" << S * NW << "] = {";
  for (int s = 0; s < S; ++s)
    for (int w = 0; w < NW; ++w)
      o << (w < (int)F.slice_roles[s].size() ? P.fwd_roles[F.slice_roles[s][w]].u0 : 0) << ",";
  o << "};\n__device__ const int kEntBegin[" << S + 1 << "] = {";
  for (int v : P.fwd_ent_begin) o << v << ",";
  o << "};\n";
  o << "extern \"C\" __global__ void __launch_bounds__((NW + 1) * 32) " << kname
    << "(const int* __restrict__ rowptr, const int* __restrict__ col, const float* __restrict__ x,\n"
       "    const float* __restrict__ Y, const float* __restrict__ W, float* __restrict__ out,\n"
       "    const int4* __restrict__ ent, const int2* __restrict__ term, int* __restrict__ err) {\n"
       "  extern __shared__ __align__(128) unsigned char smem[];\n"
       "  const int i = blockIdx.x, slice = blockIdx.y;\n"
       "  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;\n"
       "  const int e0 = rowptr[i], e1 = rowptr[i + 1];\n"
       "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
       "  if (threadIdx.x == 0) {\n"
       "    for (int s = 0; s < NSTAGE; ++s) { mbar_init(full0 + 8 * s, 32); mbar_init(empty0 + 8 * s, NW); }\n"
       "    fence_mbar_init();\n"
       "  }\n"
       "  __syncthreads();\n"
       "  if (warp == NW) { producer(col, x, Y, W, err, smem, slice, e0, e1, lane); return; }\n"
       "  const int4* sent = ent + kEntBegin[slice];\n"
       "  const int nent = kEntBegin[slice + 1] - kEntBegin[slice];\n"
       "  const int chs = slice_chs(slice);\n"
       "  const int u0 = kU0[slice * NW + warp];\n"
       "  switch (kShape[slice * NW + warp]) {\n";
  for (size_t k = 0; k < shape_rep.size(); ++k)
    o << "  case " << k << ": fcons_" << k << "(col, x, W, out, sent, nent, term, err, smem, i, e0, e1, u0, chs); break;\n";
  o << "  default: fcons_idle(sent, nent, term, err, smem, e0, e1, chs); break;\n  }\n}\n";
  return o.str();
}

cgtp_status build_forward(Plan& P) {
  // ---- roles: per hidden irrep, channel blocks x path groups
  const int kAccBudget = 64;
  P.fwd_roles.clear();
  for (size_t a = 0; a < P.in.size(); ++a) {
    const Irrep& h = P.in[a];
    std::vector<int> ps;
    for (size_t k = 0; k < P.paths.size(); ++k)
      if (P.paths[k].irrep == (int)a) ps.push_back((int)k);
    if (ps.empty()) continue;
    const int R = h.mul >= 64 ? 2 : 1;
    const int beta = std::max(13, kAccBudget / R);
    std::vector<std::vector<int>> groups;
    int sum = 0;
    for (int pi : ps) {
      const int n3 = 2 * P.paths[pi].l3 + 1;
      if (groups.empty() || sum + n3 > beta) {
        groups.push_back({});
        sum = 0;
      }
      groups.back().push_back(pi);
      sum += n3;
    }
    const int nblk = (h.mul + 32 * R - 1) / (32 * R);
    const int n1 = 2 * h.l + 1;
    for (auto& g : groups)
      for (int blk = 0; blk < nblk; ++blk) {
        FwdRole r;
        r.irrep = (int)a;
        r.u0 = blk * 32 * R;
        r.R = R;
        r.paths = g;
        double c = 0;
        for (int pi : g) c += (double)(n1 + 1) * (2 * P.paths[pi].l3 + 1);
        r.cost = c * R;
        P.fwd_roles.push_back(r);
      }
  }
  const int NR = (int)P.fwd_roles.size();
  FwdConfig& F = P.fcfg;
  F = FwdConfig();
  if (NR == 0) return CGTP_OK;  // no paths: forward writes zeros
  const int kMaxWarps = 16;
  F.S = (NR + kMaxWarps - 1) / kMaxWarps;
  // longest-processing-time assignment of roles to slices
  std::vector<int> order(NR);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return P.fwd_roles[a].cost > P.fwd_roles[b].cost; });
  const int cap = (NR + F.S - 1) / F.S;
  F.slice_roles.assign(F.S, {});
  std::vector<double> load(F.S, 0.0);
  for (int ri : order) {
    int best = -1;
    for (int s = 0; s < F.S; ++s)
      if ((int)F.slice_roles[s].size() < cap && (best < 0 || load[s] < load[best])) best = s;
    F.slice_roles[best].push_back(ri);
    load[best] += P.fwd_roles[ri].cost;
  }
  for (auto& v : F.slice_roles) std::sort(v.begin(), v.end());
  F.nw = 0;
  for (auto& v : F.slice_roles) F.nw = std::max<int>(F.nw, (int)v.size());
  F.nacc = 1;
  for (auto& r : P.fwd_roles) {
    int n = 0;
    for (int pi : r.paths) n += r.R * (2 * P.paths[pi].l3 + 1);
    F.nacc = std::max(F.nacc, n);
  }

  // ---- per-slice layouts
  std::vector<SliceLayout> SL(F.S);
  for (int s = 0; s < F.S; ++s) {
    SliceLayout& sl = SL[s];
    std::vector<char> seen(P.paths.size(), 0), iseen(P.in.size(), 0);
    for (int ri : F.slice_roles[s]) {
      for (int pi : P.fwd_roles[ri].paths) seen[pi] = 1;
      iseen[P.fwd_roles[ri].irrep] = 1;
    }
    for (size_t k = 0; k < P.paths.size(); ++k)
      if (seen[k]) {
        sl.paths.push_back((int)k);
        sl.ch_off[(int)k] = sl.chs;
        sl.chs += chat_size(P.paths[k].l1, P.paths[k].l3);
      }
    for (size_t a = 0; a < P.in.size(); ++a)
      if (iseen[a]) {
        sl.irreps.push_back((int)a);
        sl.x_st[(int)a] = sl.xs;
        sl.xs += pad4(P.in[a].mul * (2 * P.in[a].l + 1));
      }
  }
  // staging modes
  F.w_smem = (F.S == 1) && (P.U % 4 == 0);
  F.x_smem = (P.D_in % 4 == 0);
  for (int s = 0; s < F.S && F.x_smem; ++s)
    for (int a : SL[s].irreps)
      if (P.x_off[a] % 4 != 0 || (P.in[a].mul * (2 * P.in[a].l + 1)) % 4 != 0) F.x_smem = false;
  if (!F.x_smem)  // staged offsets collapse to the global ones
    for (auto& sl : SL) {
      sl.xs = 0;
      for (int a : sl.irreps) sl.x_st[a] = P.x_off[a];
    }
  // chunk size and ring depth under a shared-memory budget of ~100 KB per CTA
  int CHS = 0, XS = 0;
  for (auto& sl : SL) {
    CHS = std::max(CHS, sl.chs);
    XS = std::max(XS, sl.xs);
  }
  const long pe = (F.w_smem ? P.U * 4 : 0) + (F.x_smem ? XS * 4 : 0) + P.D_e * 4 + 64;
  const long budget = 100 * 1024;
  F.B = 4;
  while (F.B > 1 && (2L * F.B * CHS * 4 + 2L * F.B * pe) > budget) F.B /= 2;
  F.stages = (int)std::min<long>(8, std::max<long>(2, (budget - 2L * F.B * CHS * 4) / (F.B * pe)));

  cgtp_status st = upload_chat_tables(P, SL, &P.d_fwd_ent, &P.d_fwd_term, P.fwd_ent_begin);
  if (st != CGTP_OK) return st;

  int smem = 0;
  const std::string name = "cgtp_fwd";
  std::string src = gen_fwd_source(P, SL, name, smem);
  if (smem > 227 * 1024) return fail(CGTP_ERR_SIZE, "forward kernel needs too much shared memory");
  P.fwd.threads = (F.nw + 1) * 32;
  P.fwd.smem = smem;
  if (std::getenv("CGTP_DUMP_SOURCE")) {
    FILE* f = std::fopen((std::string(std::getenv("CGTP_DUMP_SOURCE")) + "/fwd.cu").c_str(), "w");
    if (f) {
      std::fputs(src.c_str(), f);
      std::fclose(f);
    }
  }
  return jit_compile(src, name, P.fwd);
}

}  // namespace cgtp
