// codegen_common.cpp -- staging layouts, the Chat tables and the two service
// warps shared by the generated forward and backward kernels.
//
// Warp organisation of both kernels (persistent CTAs; each walks the slices
// of the warp roles in turn, and in each its receivers or edge range):
//   warps 0..NW-1  consumers: pure compute on staged data
//   warp NW        TMA warp: per chunk of NB edges, bulk copies (cp.async.bulk,
//                  completion counted in bytes on the stage's "full" mbarrier)
//                  of the W and x row pieces the slice needs; pieces that are
//                  not 16-byte aligned are copied with plain loads instead.
//                  The backward's grad_out row pieces are staged once per
//                  receiver and slice, into one of two buffers.
//   warp NW+1      helper warp: loads the chunk's Y rows and builds
//                  Chat_{e,p} = sum_m2 C_p[m1][m2][m3] Y[e][m2] into the stage;
//                  in the backward it also sums the consumers' dY partials of
//                  each released stage in a fixed order and stores them.
// A stage is released ("empty" mbarrier, one arrival per consumer warp)
// after the consumers finish it.  All waits are bounded.
#include "codegen_common.hpp"

#include <algorithm>
#include <cctype>
#include <cstdlib>
#include <cstring>
#include <sstream>

namespace cgtp {

const char* kPrelude =
#include "device_prelude.inc"
    ;

std::string spin_limit_define() {
  const char* v = std::getenv("CGTP_SPIN_LIMIT");
  if (!v || !*v) return "";
  const unsigned long n = std::strtoul(v, nullptr, 10);
  return "#define CGTP_SPIN_LIMIT " + std::to_string(std::max(1ul, std::min(n, 1ul << 30))) + "u\n";
}

int max_spill_bytes(const std::string& log) {
  int best = 0;
  size_t pos = 0;
  const std::string key = " bytes spill stores";
  while ((pos = log.find(key, pos)) != std::string::npos) {
    size_t b = pos;
    while (b > 0 && std::isdigit((unsigned char)log[b - 1])) --b;
    if (b < pos) best = std::max(best, std::atoi(log.substr(b, pos - b).c_str()));
    pos += key.size();
  }
  return best;
}

int initial_min_blocks(int smem_bytes, bool* fixed) {
  if (const char* mb = std::getenv("CGTP_MIN_BLOCKS")) {
    *fixed = true;
    return std::max(1, std::atoi(mb));
  }
  *fixed = false;
  return std::max(1, std::min(3, (228 * 1024) / (smem_bytes + 1024)));
}

static void merge_segment(std::vector<Segment>& v, Segment s) {
  if (!v.empty() && v.back().src + v.back().len == s.src && v.back().dst + v.back().len == s.dst)
    v.back().len += s.len;
  else
    v.push_back(s);
}

bool segments_aligned(const std::vector<Segment>& segs, long row_len) {
  if (row_len % 4) return false;
  for (const auto& s : segs)
    if (s.src % 4 || s.dst % 4 || s.len % 4) return false;
  return true;
}

void layout_slice(const Plan& P, SliceLayout& sl, bool with_g) {
  sl.ch_off.clear();
  sl.chs = 0;
  for (int pi : sl.paths) {
    sl.ch_off[pi] = sl.chs;
    sl.chs += chat_size(P.paths[pi].l1, P.paths[pi].l3, sl.m1_major);
  }
  sl.x_st.clear();
  sl.xseg.clear();
  sl.xs = 0;
  for (int a : sl.irreps) {
    const int n = P.in[a].mul * (2 * P.in[a].l + 1);
    sl.x_st[a] = sl.xs;
    merge_segment(sl.xseg, {P.x_off[a], sl.xs, n});
    sl.xs += pad4(n);
  }
  // W pieces: every channel of every path of the slice, in column order
  std::vector<int> byk = sl.paths;
  std::sort(byk.begin(), byk.end(), [&](int a, int b) { return P.paths[a].k0 < P.paths[b].k0; });
  sl.w_st.clear();
  sl.wseg.clear();
  sl.ws = 0;
  for (int pi : byk) {
    const Path& p = P.paths[pi];
    sl.w_st[pi] = sl.ws;
    merge_segment(sl.wseg, {p.k0, sl.ws, p.mul});
    sl.ws += pad4(p.mul);
  }
  sl.g_st.clear();
  sl.gseg.clear();
  sl.gs = 0;
  if (with_g) {
    std::vector<int> byo = sl.paths;
    std::sort(byo.begin(), byo.end(), [&](int a, int b) { return P.paths[a].o_off < P.paths[b].o_off; });
    for (int pi : byo) {
      const Path& p = P.paths[pi];
      const int n = p.mul * (2 * p.l3 + 1);
      sl.g_st[pi] = sl.gs;
      merge_segment(sl.gseg, {p.o_off, sl.gs, n});
      sl.gs += pad4(n);
    }
  }
}

// Chunks ahead of the stage ring whose W rows the TMA warp prefetches into
// L2 (tuning override CGTP_PREFETCH).
static const int kDefaultPrefetch = 0;

void plan_layout(const Plan& P, const std::vector<SliceLayout>& SL, KernelShape& K, bool backward) {
  K.WS = K.XS = K.CHS = K.GS = 0;
  K.w_bulk = K.x_bulk = K.g_bulk = true;
  for (const auto& sl : SL) {
    K.WS = std::max(K.WS, sl.ws);
    K.XS = std::max(K.XS, sl.xs);
    if (!K.no_chat) K.CHS = std::max(K.CHS, sl.chs);
    K.GS = std::max(K.GS, sl.gs);
    K.w_bulk = K.w_bulk && segments_aligned(sl.wseg, P.U);
    K.x_bulk = K.x_bulk && segments_aligned(sl.xseg, P.D_in);
    K.g_bulk = K.g_bulk && segments_aligned(sl.gseg, P.D_out);
  }
  auto r128 = [](long v) { return (int)((v + 127) & ~127L); };
  const long mt = K.tangent ? 2 : 1;  // tangent kernels stage each piece twice
  auto stage_of = [&](int B) {
    long b = r128(4L * mt * B * K.WS) + r128(4L * mt * B * K.XS) + r128(4L * mt * B * P.D_e) +
             r128(4L * mt * B * K.CHS);
    if (backward) b += r128(4L * K.nw * B * P.D_e);
    return b;
  };
  // two grad_out buffers overlap the next receiver's load with this one's
  // compute; wide rows (Lmax 6) keep one so more CTAs fit
  K.gbufs = (backward && 2L * r128(4L * K.GS) > 48 * 1024) ? 1 : 2;
  const long fixed = 512 + (backward ? (long)K.gbufs * r128(4L * K.GS) : 0)  // grad_out buffers
                     + r128(4L * K.nw * K.WB);                                 // store staging
  // two or three CTAs per SM when it fits, at least two stages in flight
  // wide rows (Lmax 6) may take up to half an SM to keep two edges per chunk
  const long budget =
      std::max<long>(72 * 1024, std::min<long>(112 * 1024, fixed + 2 * stage_of(2)));
  if (K.force_B > 0) {
    K.B = K.force_B;
  } else {
    K.B = 4;
    while (K.B > 1 && fixed + 2 * stage_of(K.B) > budget) K.B /= 2;
  }
  K.stages = (int)std::min<long>(6, std::max<long>(2, (budget - fixed) / stage_of(K.B)));
  // tuning overrides: edges per chunk and ring depth
  if (const char* v = std::getenv("CGTP_CHUNK"); v && K.force_B == 0) K.B = std::max(1, std::min(8, std::atoi(v)));
  if (const char* v = std::getenv("CGTP_STAGES")) K.stages = std::max(2, std::min(6, std::atoi(v)));
  if (K.force_stages > 0) K.stages = K.force_stages;
  K.prefetch = kDefaultPrefetch;  // W rows prefetched into L2, in chunks ahead
  if (const char* v = std::getenv("CGTP_PREFETCH")) K.prefetch = std::max(0, std::min(64, std::atoi(v)));
  while (K.stages > 2 && fixed + K.stages * stage_of(K.B) > 220 * 1024) --K.stages;
  K.sdy_floats = backward ? K.nw * K.B * (int)P.D_e : 0;
  K.off_stage = 512;  // mbarriers, chunk descriptors and the edge range first
  K.off_w = 0;
  K.off_x = r128(4L * mt * K.B * K.WS);
  K.off_y = K.off_x + r128(4L * mt * K.B * K.XS);
  K.off_ch = K.off_y + r128(4L * mt * K.B * P.D_e);
  K.off_dy = K.off_ch + r128(4L * mt * K.B * K.CHS);
  K.stage_bytes = K.off_dy + (backward ? r128(4L * K.sdy_floats) : 0);
  K.off_g = K.off_stage + K.stages * K.stage_bytes;
  K.off_wb = K.off_g + (backward ? K.gbufs * r128(4L * K.GS) : 0);
  K.smem = K.off_wb + r128(4L * K.nw * K.WB);
}

// bulk-or-plain copy of row pieces for the edges of a chunk.  Bulk copies are
// issued by lane b for edge b; plain copies are spread over the warp.
static void gen_copy_pieces(std::ostringstream& o, const std::vector<Segment>& segs, bool bulk,
                            const std::string& dst_row /* float* of edge 0 */, int stride,
                            const std::string& src_row /* expression of b */, const std::string& bar,
                            bool one_block, long row_len) {
  if (bulk && one_block) {
    // staged rows identical to the global rows: one copy for the chunk
    o << "      if (lane == 0) bulk_g2s_stream(smem_u32(" << dst_row << "), " << src_row
      << "(0), (u32)nb * " << row_len * 4 << ", " << bar << ", pol);\n";
    return;
  }
  if (bulk) {
    o << "      if (lane < nb) {\n        const int b = lane;\n";
    for (const auto& s : segs)
      o << "        bulk_g2s(smem_u32(" << dst_row << " + b * " << stride << " + " << s.dst << "), " << src_row
        << "(b) + " << s.src << ", " << s.len * 4 << ", " << bar << ");\n";
    o << "      }\n";
    return;
  }
  for (const auto& s : segs)
    o << "      for (int t = lane; t < nb * " << s.len << "; t += 32) { const int b = t / " << s.len
      << ", q = t - b * " << s.len << "; " << dst_row << "[b * " << stride << " + " << s.dst << " + q] = "
      << src_row << "(b)[" << s.src << " + q]; }\n";
}

std::string gen_common_device(const Plan& P, const std::vector<SliceLayout>& SL, const KernelShape& K,
                              bool backward) {
  std::ostringstream o;
  const int S = K.S;
  o << "#define NW " << K.nw << "\n#define NB " << K.B << "\n#define NSTAGE " << K.stages
    << "\n#define NSLICE " << S << "\n#define DIN " << P.D_in << "\n#define DE " << P.D_e
    << "\n#define DOUT " << P.D_out << "\n#define NU " << P.U << "\n#define WS " << K.WS
    << "\n#define XS " << K.XS << "\n#define CHS " << K.CHS << "\n#define STAGE_BYTES " << K.stage_bytes
    << "\n#define OFF_STAGE " << K.off_stage << "\n#define OFF_W " << K.off_w << "\n#define OFF_X "
    << K.off_x << "\n#define OFF_Y " << K.off_y << "\n#define OFF_CH " << K.off_ch << "\n#define OFF_DY "
    << K.off_dy << "\n#define OFF_G " << K.off_g << "\n#define GS " << K.GS << "\n#define WB " << K.WB
    << "\n#define OFF_WB " << K.off_wb << "\n#define FULL_COUNT 32\n#define CHAT_COUNT 32\n#define GBUF " << K.gbufs << "\n#define YPL "
    << (K.B * P.D_e + 31) / 32 << "\n#define TAN " << (K.tangent ? 1 : 0) << "\n#define PF " << K.prefetch
    << "\n";
  // tangent copies of a stage's regions, right after the plain ones
  o << "#define OFF_WT (OFF_W + 4 * NB * WS)\n#define OFF_XT (OFF_X + 4 * NB * XS)\n"
       "#define OFF_YT (OFF_Y + 4 * NB * DE)\n#define OFF_CHT (OFF_CH + 4 * NB * CHS)\n";
  // shared-memory header: full[NSTAGE] (the TMA warp's 32 lanes and the
  // bytes of its copies), empty[NSTAGE] (one arrival per consumer warp),
  // chat[NSTAGE] (the helper's 32 lanes: Y and Chat of the stage written),
  // gfull[2], gempty[2] mbarriers, the helper's per-stage chunk descriptors,
  // and the edge range of the edge-range variant, all below OFF_STAGE
  // (mbarriers 8-byte aligned; the int4 descriptors and range 16-byte aligned)
  {
    const int off_chat = 2 * K.stages * 8;
    const int off_gfull = (3 * K.stages * 8 + 15) & ~15;
    const int off_gempty = off_gfull + 16;
    const int off_desc = off_gempty + 16;
    const int off_range = off_desc + 16 * K.stages;
    o << "#define OFF_CHAT " << off_chat << "\n#define OFF_GFULL " << off_gfull << "\n#define OFF_GEMPTY "
      << off_gempty << "\n#define OFF_DESC " << off_desc << "\n#define OFF_RANGE " << off_range << "\n";
  }
  // a stage is ready for the consumers when its copies have landed and its
  // Chat is built
  o << "__device__ __forceinline__ bool stage_ready(u32 full0, int s, u32 parity) {\n"
       "  return mbar_wait(full0 + 8 * s, parity) && mbar_wait(full0 + OFF_CHAT + 8 * s, parity);\n}\n";
  // the receivers a CTA walks: whole receivers blockIdx.x, + gridDim.x, ...,
  // or (backward, edge_ranges) an equal share of the edges, receivers clipped
  // to it (the range sits in the header at OFF_RANGE)
  if (backward && K.edge_ranges)
    o << "#define RANGE_AT(k) (reinterpret_cast<const int*>(smem + OFF_RANGE)[k])\n"
         "#define RECV_FIRST RANGE_AT(0)\n#define RECV_END RANGE_AT(1)\n#define RECV_STEP 1\n"
         "#define EDGE_LO(i) max(rowptr[i], RANGE_AT(2))\n#define EDGE_HI(i) min(rowptr[(i) + 1], RANGE_AT(3))\n";
  else
    o << "#define RECV_FIRST ((int)blockIdx.x)\n#define RECV_END n_recv\n#define RECV_STEP ((int)gridDim.x)\n"
         "#define EDGE_LO(i) rowptr[i]\n#define EDGE_HI(i) rowptr[(i) + 1]\n";
  if (backward) {
    o << "__constant__ int kPh[" << S * K.nw << "] = {";
    for (int s = 0; s < S; ++s)
      for (int w = 0; w < K.nw; ++w) {
        const auto& v = P.bcfg.slice_roles[s];
        o << (w < (int)v.size() ? P.bwd_roles[v[w]].ph : -1) << ",";
      }
    o << "};\n__constant__ int kNph[" << S * K.nw << "] = {";
    for (int s = 0; s < S; ++s)
      for (int w = 0; w < K.nw; ++w) {
        const auto& v = P.bcfg.slice_roles[s];
        o << (w < (int)v.size() ? P.bwd_roles[v[w]].nph : 1) << ",";
      }
    o << "};\n";
  }
  o << "__constant__ int kChs[" << S << "] = {";
  for (int s = 0; s < S; ++s) o << SL[s].chs << ",";
  o << "};\n";
  o << "__device__ __forceinline__ unsigned char* stage_ptr(unsigned char* smem, int s) {\n"
       "  return smem + OFF_STAGE + s * STAGE_BYTES;\n}\n";

  // ---- TMA warp.  Every warp of a CTA walks the same sequence: for each
  // slice in order, the receivers blockIdx.x, + gridDim.x, ..., and their
  // chunks; the running chunk counter q picks the stage and the phase.
  // eid (nullable): the edges' ids in the full edge set, whose W rows the
  // chunk reads (the sparse evaluation's active edges); NULL: W row = edge
  // xt, Wt: the tangent inputs of tangent kernels (unused otherwise)
  o << "__device__ __noinline__ void tma_warp(const int* __restrict__ rowptr, int n_recv,\n"
       "    const int* __restrict__ col, const float* __restrict__ x, const float* __restrict__ W,\n"
       "    const float* __restrict__ xt, const float* __restrict__ Wt,\n"
       "    const int* __restrict__ eid, const float* __restrict__ g, int* __restrict__ err,\n"
       "    unsigned char* smem, int lane) {\n"
       "  (void)xt; (void)Wt;\n"
       "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
       "  const u32 gfull0 = full0 + OFF_GFULL, gempty0 = full0 + OFF_GEMPTY;\n"
       "  (void)gfull0; (void)gempty0; (void)g;\n"
       "  const u64 pol = policy_evict_first();\n"
       "  (void)pol;\n"
       "  int q = 0, k = 0;  // chunks and grad_out loads issued\n"
       "  (void)k;\n"
       "  bool dead = false;\n"
       "  for (int slice = 0; slice < NSLICE && !dead; ++slice) {\n"
       "  // The receivers' edge ranges are loaded two receivers ahead and their\n"
       "  // first 32 sender ids (one per lane) one receiver ahead, so that no\n"
       "  // chunk waits on a dependent global load before its copies are issued.\n"
       "  int e0n = 0, e1n = 0, e0nn = 0, e1nn = 0, cnext = 0;\n"
       "  if (RECV_FIRST < RECV_END) {\n"
       "    e0n = EDGE_LO(RECV_FIRST); e1n = EDGE_HI(RECV_FIRST);\n"
       "    cnext = (e0n + lane < e1n) ? __ldg(col + e0n + lane) : 0;\n"
       "    if (RECV_FIRST + RECV_STEP < RECV_END) { e0nn = EDGE_LO(RECV_FIRST + RECV_STEP); e1nn = EDGE_HI(RECV_FIRST + RECV_STEP); }\n"
       "  }\n"
       "  for (int i = RECV_FIRST; i < RECV_END && !dead; i += RECV_STEP) {\n"
       "    const int e0 = e0n, e1 = e1n;\n"
       "    int cbase = e0, cwin = cnext;  // sender ids of edges [cbase, cbase + 32), one per lane\n"
       "    e0n = e0nn; e1n = e1nn;\n"
       "    cnext = (i + RECV_STEP < RECV_END && e0n + lane < e1n) ? __ldg(col + e0n + lane) : 0;\n"
       "    if (i + 2 * RECV_STEP < RECV_END) { e0nn = EDGE_LO(i + 2 * RECV_STEP); e1nn = EDGE_HI(i + 2 * RECV_STEP); }\n"
       "    (void)cbase; (void)cwin;\n";
  if (backward) o << "    if (e1 <= e0) continue;\n";
  o << "    switch (slice) {\n";
  for (int s = 0; s < S; ++s) {
    const SliceLayout& sl = SL[s];
    long wb = 0, xb = 0, gb = 0;
    for (auto& q : sl.wseg) wb += q.len * 4;
    for (auto& q : sl.xseg) xb += q.len * 4;
    for (auto& q : sl.gseg) gb += q.len * 4;
    const bool w_one = sl.wseg.size() == 1 && sl.wseg[0].src == 0 && sl.wseg[0].dst == 0 &&
                       sl.wseg[0].len == P.U && sl.ws == P.U;
    o << "    case " << s << ": {\n";
    if (backward) {
      o << "      {  // this receiver's grad_out pieces into buffer k % GBUF\n"
           "        const int gb = k % GBUF;\n"
           "        if (k >= GBUF && !mbar_wait(gempty0 + 8 * gb, ((k / GBUF) - 1) & 1)) { if (lane == 0) atomicOr(err, 10); dead = true; break; }\n"
           "        float* sg = reinterpret_cast<float*>(smem + OFF_G) + gb * GS;\n"
           "        const float* grow = g + (size_t)i * DOUT;\n";
      if (K.g_bulk) {
        o << "        if (lane == 0) {\n          mbar_expect_tx(gfull0 + 8 * gb, " << gb << ");\n";
        for (auto& q : sl.gseg)
          o << "          bulk_g2s(smem_u32(sg + " << q.dst << "), grow + " << q.src << ", " << q.len * 4
            << ", gfull0 + 8 * gb);\n";
        o << "        }\n";
      } else {
        for (auto& q : sl.gseg)
          o << "        for (int t = lane; t < " << q.len << "; t += 32) sg[" << q.dst << " + t] = grow["
            << q.src << " + t];\n";
      }
      o << "        mbar_arrive(gfull0 + 8 * gb);\n"
           "        ++k;\n      }\n";
    }
    // W rows PF chunks ahead (into the CTA's next receiver near the end of
    // this one) are prefetched into L2 before the wait for a free stage
    std::ostringstream pf;
    if (K.prefetch > 0 && K.w_bulk) {
      pf << "        {\n"
            "          int pe = eb + PF * NB, pe1 = e1;\n"
            "          if (pe >= e1) {  // past this receiver: the next one's edges\n"
            "            const int i2 = i + RECV_STEP;\n"
            "            pe1 = 0;\n"
            "            if (i2 < RECV_END) { const int a2 = EDGE_LO(i2); pe1 = EDGE_HI(i2); pe = a2 + (pe - e1); }\n"
            "          }\n"
            "          const int npf = min(NB, pe1 - pe);\n"
            "          if (npf > 0) {\n";
      if (w_one)
        pf << "            if (eid == nullptr) {\n"
              "              if (lane == 0) bulk_prefetch_l2(W + (size_t)pe * NU, (u32)npf * " << P.U * 4 << ");\n"
              "            } else if (lane < npf) {\n"
              "              bulk_prefetch_l2(W + (size_t)__ldg(eid + pe + lane) * NU, " << P.U * 4 << ");\n"
              "            }\n";
      else {
        pf << "            if (lane < npf) {\n"
              "              const float* wrow = W + (size_t)(eid ? __ldg(eid + pe + lane) : pe + lane) * NU;\n";
        for (auto& q : sl.wseg) pf << "              bulk_prefetch_l2(wrow + " << q.src << ", " << q.len * 4 << ");\n";
        pf << "            }\n";
      }
      pf << "          }\n        }\n";
    }
    o << "      for (int eb = e0; eb < e1; eb += NB, ++q) {\n"
         "        const int s = q % NSTAGE;\n"
         "        const int nb = min(NB, e1 - eb);\n"
         "        if (eb + nb > cbase + 32) {  // the next 32 sender ids of this receiver\n"
         "          cbase = eb;\n"
         "          cwin = (eb + lane < e1) ? __ldg(col + eb + lane) : 0;\n"
         "        }\n"
         "        const int jj = __shfl_sync(0xffffffffu, cwin, (eb - cbase + lane) & 31);  // edge eb + lane's sender\n"
      << pf.str();
    o << ""
         "        if (q >= NSTAGE && !mbar_wait(empty0 + 8 * s, ((q / NSTAGE) - 1) & 1)) { if (lane == 0) atomicOr(err, 10); dead = true; break; }\n"
         "        unsigned char* st = stage_ptr(smem, s);\n"
         "        float* sW = reinterpret_cast<float*>(st + OFF_W);\n"
         "        float* sX = reinterpret_cast<float*>(st + OFF_X);\n"
         "        float* sWt = reinterpret_cast<float*>(st + OFF_WT);\n"
         "        float* sXt = reinterpret_cast<float*>(st + OFF_XT);\n"
         "        (void)sW; (void)sX; (void)sWt; (void)sXt;\n"
         "        (void)jj;\n"
         "        if (lane == 0) mbar_expect_tx(full0 + 8 * s, (u32)nb * "
      << (K.tangent ? 2 : 1) * ((K.w_bulk ? wb : 0) + (K.x_bulk ? xb : 0)) << ");\n"
      << "        __syncwarp();\n";
    std::ostringstream cp;
    // W rows: consecutive for a chunk of one receiver's edges, or (eid) the
    // rows of the listed edges, one copy per edge
    cp << "if (eid == nullptr) {\n#define WROW(b) (W + (size_t)(eb + (b)) * NU)\n";
    gen_copy_pieces(cp, sl.wseg, K.w_bulk, "sW", K.WS, "WROW", "full0 + 8 * s", w_one, P.U);
    cp << "#undef WROW\n";
    if (K.tangent) {
      cp << "#define WTROW(b) (Wt + (size_t)(eb + (b)) * NU)\n";
      gen_copy_pieces(cp, sl.wseg, K.w_bulk, "sWt", K.WS, "WTROW", "full0 + 8 * s", w_one, P.U);
      cp << "#undef WTROW\n";
    }
    cp << "} else {\n#define WROW(b) (W + (size_t)__ldg(eid + eb + (b)) * NU)\n";
    gen_copy_pieces(cp, sl.wseg, K.w_bulk, "sW", K.WS, "WROW", "full0 + 8 * s", false, P.U);
    cp << "#undef WROW\n";
    if (K.tangent) {
      cp << "#define WTROW(b) (Wt + (size_t)__ldg(eid + eb + (b)) * NU)\n";
      gen_copy_pieces(cp, sl.wseg, K.w_bulk, "sWt", K.WS, "WTROW", "full0 + 8 * s", false, P.U);
      cp << "#undef WTROW\n";
    }
    cp << "}\n";
    if (K.x_bulk) {
      cp << "#define XROW(b) (x + (size_t)jj * DIN)\n";
      gen_copy_pieces(cp, sl.xseg, true, "sX", K.XS, "XROW", "full0 + 8 * s", false, P.D_in);
      if (K.tangent) {
        cp << "#define XTROW(b) (xt + (size_t)jj * DIN)\n";
        gen_copy_pieces(cp, sl.xseg, true, "sXt", K.XS, "XTROW", "full0 + 8 * s", false, P.D_in);
        cp << "#undef XTROW\n";
      }
    } else {
      cp << "#define XROW(b) (x + (size_t)col[eb + (b)] * DIN)\n";
      gen_copy_pieces(cp, sl.xseg, false, "sX", K.XS, "XROW", "full0 + 8 * s", false, P.D_in);
      if (K.tangent) {
        cp << "#define XTROW(b) (xt + (size_t)col[eb + (b)] * DIN)\n";
        gen_copy_pieces(cp, sl.xseg, false, "sXt", K.XS, "XTROW", "full0 + 8 * s", false, P.D_in);
        cp << "#undef XTROW\n";
      }
    }
    cp << "#undef XROW\n";
    std::string c = cp.str(), ind;
    size_t pos = 0;
    while (pos < c.size()) {
      size_t e = c.find('\n', pos);
      if (e == std::string::npos) e = c.size();
      std::string line = c.substr(pos, e - pos);
      ind += (line.rfind("#", 0) == 0 ? "" : "  ") + line + "\n";
      pos = e + 1;
    }
    o << ind
      << "        mbar_arrive(full0 + 8 * s);\n"
         "      }\n"
         "      break;\n    }\n";
  }
  o << "    }\n"
       "  }\n"
       "  }\n"
       "  // every bulk copy this warp issued must land before the CTA may exit:\n"
       "  // the last NSTAGE chunks' and the last GBUF grad_out loads' barriers\n"
       "  // complete on this warp's own arrivals and bytes alone\n"
       "  if (lane == 0) {\n"
       "    for (int c = max(0, q - NSTAGE); c < q; ++c)\n"
       "      if (!mbar_wait_drain(full0 + 8 * (c % NSTAGE), (c / NSTAGE) & 1)) atomicOr(err, 10);\n";
  if (backward)
    o << "    for (int c = max(0, k - GBUF); c < k; ++c)\n"
         "      if (!mbar_wait_drain(gfull0 + 8 * (c % GBUF), (c / GBUF) & 1)) atomicOr(err, 10);\n";
  o << "  }\n"
       "}\n";

  // ---- helper warp
  if (backward) {
    o << "__device__ __forceinline__ void reduce_dy(unsigned char* smem, int s, int4 d, float* __restrict__ dyp,\n"
         "    int E, int lane) {\n"
         "  // d = (first edge, edges, slice) of the chunk that stage s held\n"
         "  const float* sdy = reinterpret_cast<const float*>(stage_ptr(smem, s) + OFF_DY);\n"
         "  float* dys = dyp + (size_t)d.z * E * DE;\n"
         "  for (int t = lane; t < d.y * DE; t += 32) {\n"
         "    const int b = t / DE, k = t - b * DE;\n"
         "    float v = 0.f;\n"
         "#pragma unroll\n"
         "    for (int w = 0; w < NW; ++w) {\n"
         "      const int ph = kPh[d.z * NW + w];\n"
         "      if (ph >= 0 && (b & (kNph[d.z * NW + w] - 1)) == ph) v += sdy[(w * NB + b) * DE + k];\n"
         "    }\n"
         "    dys[(size_t)(d.x + b) * DE + k] = v;\n"
         "  }\n"
         "}\n";
  }
  // Yt: the tangent harmonics of tangent kernels (unused otherwise)
  // E (backward): the edge stride between the slices' dY parts, the host's
  // edge count (for the sparse evaluation an upper bound of the compact
  // count the device CSR holds)
  o << "__device__ __noinline__ void helper_warp(const int* __restrict__ rowptr, int n_recv,\n"
       "    const float* __restrict__ Y, const float* __restrict__ Yt, const int4* __restrict__ rec,\n"
       "    const int* __restrict__ rec_begin, float* __restrict__ dyp, int* __restrict__ err,\n"
       "    unsigned char* smem, int lane, int E) {\n"
       "  (void)Yt;\n"
       "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
       "  int4* desc = reinterpret_cast<int4*>(smem + OFF_DESC);  // (eb, nb, slice, -) of each stage\n"
       "  (void)dyp; (void)desc;\n"
       "  (void)E;\n"
       "  int last_slice[NSTAGE];\n"
       "#pragma unroll\n"
       "  for (int s = 0; s < NSTAGE; ++s) last_slice[s] = -1;\n"
       "  int q = 0;\n"
       "  bool dead = false;\n"
       "  for (int slice = 0; slice < NSLICE && !dead; ++slice) {\n"
       "  const int chs = kChs[slice];\n"
       "  const int4* srec = rec + rec_begin[slice];\n"
       "  const int nrec = rec_begin[slice + 1] - rec_begin[slice];\n"
       "  (void)srec; (void)nrec;\n";
  const int KR = (K.rec_max + 31) / 32;
  const bool rec_regs = KR <= 12;
  if (rec_regs && !K.no_chat)  // the slice's records stay in registers: no loads in the Chat loop
    o << "  int rd[" << KR << "];\n  float rc0[" << KR << "], rc1[" << KR << "];\n"
      << "  const int nk = (nrec - lane + 31) >> 5;\n"
      << "#pragma unroll\n  for (int k = 0; k < " << KR << "; ++k) {\n"
      << "    const int4 r = k < nk ? __ldg(srec + lane + 32 * k) : make_int4(0, 0, 0, 0);\n"
      << "    rd[k] = r.x;\n    rc0[k] = __int_as_float(r.y);\n    rc1[k] = __int_as_float(r.z);\n  }\n";
  o <<
       "  for (int i = RECV_FIRST; i < RECV_END && !dead; i += RECV_STEP) {\n"
       "    const int e0 = EDGE_LO(i), e1 = EDGE_HI(i);\n"
       "    for (int eb = e0; eb < e1; eb += NB, ++q) {\n"
       "      const int s = q % NSTAGE;\n"
       "      const int nb = min(NB, e1 - eb);\n"
       "      // this chunk's Y values travel while the stage is still in use\n"
       "      float yv[YPL], ytv[TAN ? YPL : 1];\n"
       "      (void)ytv;\n"
       "#pragma unroll\n"
       "      for (int k = 0; k < YPL; ++k) { const int t = lane + 32 * k; yv[k] = t < nb * DE ? __ldg(Y + (size_t)eb * DE + t) : 0.f; }\n"
       "#if TAN\n"
       "#pragma unroll\n"
       "      for (int k = 0; k < YPL; ++k) { const int t = lane + 32 * k; ytv[k] = t < nb * DE ? __ldg(Yt + (size_t)eb * DE + t) : 0.f; }\n"
       "#endif\n"
       "      if (q >= NSTAGE) {\n"
       "        if (!mbar_wait(empty0 + 8 * s, ((q / NSTAGE) - 1) & 1)) { if (lane == 0) atomicOr(err, 10); dead = true; break; }\n";
  if (backward)
    o << "        if (dyp) { __syncwarp(); reduce_dy(smem, s, desc[s], dyp, E, lane); }\n";
  o << "      }\n"
       "      unsigned char* st = stage_ptr(smem, s);\n"
       "      float* sY = reinterpret_cast<float*>(st + OFF_Y);\n"
       "      float* ch = reinterpret_cast<float*>(st + OFF_CH);\n"
       "      bool fresh = false;\n"
       "#pragma unroll\n"
       "      for (int t = 0; t < NSTAGE; ++t)\n"
       "        if (t == s && last_slice[t] != slice) { last_slice[t] = slice; fresh = true; }\n"
       "      float* sYt = reinterpret_cast<float*>(st + OFF_YT);\n"
       "      float* cht = reinterpret_cast<float*>(st + OFF_CHT);\n"
       "      (void)sYt; (void)cht;\n"
    << (K.no_chat ? "      (void)fresh; (void)ch;\n"
                  : "      if (fresh)  // Chat elements without a CG term are zero for this slice\n"
                    "        for (int t = lane; t < (TAN ? 2 : 1) * NB * CHS; t += 32) ch[t] = 0.f;\n")
    <<
       "#pragma unroll\n"
       "      for (int k = 0; k < YPL; ++k) { const int t = lane + 32 * k; if (t < nb * DE) sY[t] = yv[k]; }\n"
       "#if TAN\n"
       "#pragma unroll\n"
       "      for (int k = 0; k < YPL; ++k) { const int t = lane + 32 * k; if (t < nb * DE) sYt[t] = ytv[k]; }\n"
       "#endif\n"
       "      if (lane == 0) desc[s] = make_int4(eb, nb, slice, 0);\n"
       "      __syncwarp();\n"
       "";
  if (K.no_chat)
    ;  // the consumers contract with the CG table and Y directly
  else if (rec_regs)
    o << "#pragma unroll\n"
         "      for (int k = 0; k < " << KR << "; ++k) {\n"
         "        if (k < nk) {\n"
         "          const int d = rd[k] & 0xffff, ia = (rd[k] >> 16) & 0xff, ib = (unsigned)rd[k] >> 24;\n"
         "#pragma unroll\n"
         "          for (int b = 0; b < NB; ++b)\n"
         "            if (b < nb) {\n"
         "              ch[b * chs + d] = fmaf(rc0[k], sY[b * DE + ia], rc1[k] * sY[b * DE + ib]);\n"
         "#if TAN\n"
         "              cht[b * chs + d] = fmaf(rc0[k], sYt[b * DE + ia], rc1[k] * sYt[b * DE + ib]);\n"
         "#endif\n"
         "            }\n"
         "        }\n"
         "      }\n";
  else
    o << "      for (int b = 0; b < nb; ++b) {\n"
         "        const float* y = sY + b * DE;\n"
         "        float* cb = ch + b * chs;\n"
         "#pragma unroll 4\n"
         "        for (int r0 = lane; r0 < nrec; r0 += 32) {\n"
         "          const int4 r = __ldg(srec + r0);\n"
         "          cb[r.x & 0xffff] = fmaf(__int_as_float(r.y), y[(r.x >> 16) & 0xff], __int_as_float(r.z) * y[(unsigned)r.x >> 24]);\n"
         "#if TAN\n"
         "          cht[b * chs + (r.x & 0xffff)] = fmaf(__int_as_float(r.y), sYt[b * DE + ((r.x >> 16) & 0xff)],\n"
         "                                              __int_as_float(r.z) * sYt[b * DE + ((unsigned)r.x >> 24)]);\n"
         "#endif\n"
         "        }\n"
         "      }\n";
  o << "      mbar_arrive(full0 + OFF_CHAT + 8 * s);\n"
       "    }\n"
       "  }\n"
       "  }\n";
  if (backward)
    o << "  if (!dead && dyp)\n"
         "    for (int c = max(0, q - NSTAGE); c < q; ++c) {\n"
         "      const int s = c % NSTAGE;\n"
         "      if (!mbar_wait(empty0 + 8 * s, (c / NSTAGE) & 1)) { if (lane == 0) atomicOr(err, 10); break; }\n"
         "      __syncwarp();\n"
         "      reduce_dy(smem, s, desc[s], dyp, E, lane);\n"
         "    }\n";
  o << "}\n";
  return o.str();
}

// One 16-byte record per non-zero Chat element of a slice's paths (real CG
// blocks have at most two non-zero C[m1][m2][m3] for a given (m1, m3)):
//   x = dst offset in the edge's Chat block | y0 << 16 | y1 << 24
//   y = coefficient of Y[y0], z = coefficient of Y[y1] (FP32 bits), w = 0.
// Elements with no term stay zero: the helper clears the Chat buffers once.
cgtp_status upload_chat_tables(const Plan& P, const std::vector<SliceLayout>& SL, void** d_ent,
                               std::vector<int>& ent_begin) {
  std::vector<int> rec;
  ent_begin.assign(1, 0);
  for (const SliceLayout& sl : SL) {
    for (int pi : sl.paths) {
      const Path& p = P.paths[pi];
      const int n1 = 2 * p.l1 + 1, n2 = 2 * p.l2 + 1, n3 = 2 * p.l3 + 1;
      const double* C = P.coeff.data() + p.c_off;
      for (int m3 = 0; m3 < n3; ++m3)
        for (int m1 = 0; m1 < n1; ++m1) {
          int yi[2] = {0, 0};
          float cf[2] = {0.f, 0.f};
          int cnt = 0;
          for (int m2 = 0; m2 < n2; ++m2) {
            const double c = C[((size_t)m1 * n2 + m2) * n3 + m3];
            if (c == 0.0) continue;
            if (cnt == 2) return fail(CGTP_ERR_SIZE, "a Chat element with more than two CG terms");
            yi[cnt] = p.l2 * p.l2 + m2;
            cf[cnt] = (float)c;
            ++cnt;
          }
          if (cnt == 0) continue;
          const int dst = sl.ch_off.at(pi) + chat_pos(p.l1, p.l3, m1, m3, sl.m1_major);
          if (dst >= (1 << 16) || yi[0] >= 256 || yi[1] >= 256)
            return fail(CGTP_ERR_SIZE, "Chat block too large for the record format");
          int b0, b1;
          std::memcpy(&b0, &cf[0], 4);
          std::memcpy(&b1, &cf[1], 4);
          rec.push_back(dst | (yi[0] << 16) | (yi[1] << 24));
          rec.push_back(b0);
          rec.push_back(b1);
          rec.push_back(0);
        }
    }
    ent_begin.push_back((int)rec.size() / 4);
  }
  if (P.host_only) return CGTP_OK;
  if (rec.empty()) rec.assign(4, 0);
  if (cudaMalloc(d_ent, rec.size() * sizeof(int)) != cudaSuccess)
    return fail(CGTP_ERR_OOM, "cudaMalloc of the Chat tables");
  CGTP_CUDA_TRY(cudaMemcpy(*d_ent, rec.data(), rec.size() * sizeof(int), cudaMemcpyHostToDevice));
  return CGTP_OK;
}

}  // namespace cgtp
