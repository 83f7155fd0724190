// codegen_common.hpp -- pieces shared by the forward and backward code
// generators: the device prelude, per-slice staging layouts, the Chat tables,
// and the two service warps of both kernels.
#pragma once

#include <map>
#include <string>
#include <vector>

#include "internal.hpp"

namespace cgtp {

extern const char* kPrelude;

// "#define CGTP_SPIN_LIMIT n" when the CGTP_SPIN_LIMIT environment variable
// is set at plan creation (a smaller bound for the pipeline waits, for tests
// of the kernels' wind-down after an expired wait), else "".
std::string spin_limit_define();

inline int pad4(int n) { return (n + 3) & ~3; }

// Chat_{e,p} = sum_m2 C_p[m1][m2][m3] Y[e][l2^2+m2], stored per edge and path
// as [N3][pad4(N1)] (m3-major) or [N1][pad4(N3)] (m1-major, rows of m3 pairs
// for the packed forward) when N1 > 1, and as one padded row [pad4(N3)] when
// N1 == 1.
inline int chat_size(int l1, int l3, bool m1_major) {
  const int n1 = 2 * l1 + 1, n3 = 2 * l3 + 1;
  return n1 == 1 ? pad4(n3) : m1_major ? n1 * pad4(n3) : n3 * pad4(n1);
}
inline int chat_pos(int l1, int l3, int m1, int m3, bool m1_major) {
  const int n1 = 2 * l1 + 1, n3 = 2 * l3 + 1;
  return n1 == 1 ? m3 : m1_major ? m1 * pad4(n3) + m3 : m3 * pad4(n1) + m1;
}

// A contiguous piece of a global row copied into a staged row.
struct Segment {
  int src;  // float offset in the global row
  int dst;  // float offset in the staged row
  int len;  // floats
};

struct SliceLayout {
  bool m1_major = false;       // Chat layout (see chat_pos)
  std::vector<int> paths;      // paths whose Chat the slice needs
  std::map<int, int> ch_off;   // path -> Chat offset (floats, per edge)
  int chs = 0;                 // Chat floats per edge
  std::vector<int> irreps;     // hidden irreps of the slice
  std::map<int, int> x_st;     // irrep -> staged x offset
  std::vector<Segment> xseg;   // x row pieces
  int xs = 0;                  // staged x floats per edge
  std::map<int, int> w_st;     // path -> staged W offset of its channel 0
  std::vector<Segment> wseg;   // W row pieces
  int ws = 0;                  // staged W floats per edge
  std::map<int, int> g_st;     // path -> staged grad_out offset (backward)
  std::vector<Segment> gseg;   // grad_out row pieces (backward)
  int gs = 0;                  // staged grad_out floats per receiver
};

// Builds the staging layout of one slice from its paths and irreps.
void layout_slice(const Plan& P, SliceLayout& sl, bool with_g);

// Whether every piece of the slice can move by bulk copy (16-byte aligned
// starts and lengths in both the global and the staged row).
bool segments_aligned(const std::vector<Segment>& segs, long row_len);

struct KernelShape {
  int S = 1, nw = 0, B = 2, stages = 3;
  bool w_bulk = true, x_bulk = true, g_bulk = true;
  int WS = 0, XS = 0, CHS = 0, GS = 0;
  int sdy_floats = 0;  // per stage (backward)
  // byte offsets in dynamic shared memory
  int off_stage = 0, stage_bytes = 0, off_w = 0, off_x = 0, off_y = 0, off_ch = 0, off_dy = 0;
  int off_g = 0, smem = 0;
  int WB = 0;       // per-consumer-warp staging buffer for coalesced row stores (floats)
  int gbufs = 2;    // grad_out row buffers (backward)
  int force_B = 0;  // edges per chunk fixed by the caller (0: chosen from the budget)
  int force_stages = 0;  // ring depth fixed by the caller (0: chosen from the budget)
  int rec_max = 0;  // most Chat records of a slice
  bool edge_ranges = false;  // backward CTAs take equal edge ranges
  // tangent kernels: every staged W, x and Y piece (and so Chat) has a
  // second copy holding its directional derivative (the double backward)
  bool tangent = false;
  // forward: add the result to the output rows instead of writing them
  bool accumulate = false;
  // W rows prefetched into L2 this many chunks ahead (0: off)
  int prefetch = 0;
  // forward roles with float2 accumulators of m3 pairs and packed FMAs over
  // an m1-major Chat (fpath2, fpath_tan2)
  bool packed = false;
  // backward roles that contract with the CG table and Y directly: no Chat
  // is staged or built (the default; CGTP_BWD_TFORM=0 turns it off)
  bool no_chat = false;
  int off_wb = 0;
};

// Fills the shared-memory layout of a kernel; extra per-stage floats for the
// backward's dY partials.
void plan_layout(const Plan& P, const std::vector<SliceLayout>& SL, KernelShape& K, bool backward);

// Device code: #defines, per-slice staging switches, the TMA warp and the
// helper warp.  (backward: grad_out staging and dY reduction.)
std::string gen_common_device(const Plan& P, const std::vector<SliceLayout>& SL,
                              const KernelShape& K, bool backward);

// Largest "N bytes spill stores" of a compiler log.
int max_spill_bytes(const std::string& log);

// Resident CTAs per SM the shared memory allows (at most 3): the starting
// point of the register cap; CGTP_MIN_BLOCKS overrides it.
int initial_min_blocks(int smem_bytes, bool* fixed);

// The Chat records of every slice (16 bytes each: target | y index a |
// y index b, c_a, c_b) uploaded to the device; ent_begin[s] is slice s's first.
cgtp_status upload_chat_tables(const Plan& P, const std::vector<SliceLayout>& SL, void** d_ent,
                               std::vector<int>& ent_begin);

}  // namespace cgtp
