// codegen_common.hpp -- pieces shared by the forward and backward code
// generators: the device prelude, the per-edge Chat layout and its tables.
#pragma once

#include <map>
#include <string>
#include <vector>

#include "internal.hpp"

namespace cgtp {

extern const char* kPrelude;

inline int pad4(int n) { return (n + 3) & ~3; }

// Chat_{e,p} = sum_m2 C_p[m1][m2][m3] Y[e][l2^2+m2], stored per edge and path
// as [N3][pad4(N1)] when N1 > 1 and as one padded row [pad4(N3)] when N1 == 1.
inline int chat_size(int l1, int l3) {
  const int n1 = 2 * l1 + 1, n3 = 2 * l3 + 1;
  return n1 == 1 ? pad4(n3) : n3 * pad4(n1);
}
inline int chat_pos(int l1, int l3, int m1, int m3) {
  const int n1 = 2 * l1 + 1;
  return n1 == 1 ? m3 : m3 * pad4(n1) + m1;
}

struct SliceLayout {
  std::vector<int> paths;     // unique paths of the slice
  std::map<int, int> ch_off;  // path -> Chat offset (floats)
  int chs = 0;                // Chat floats per edge
  std::vector<int> irreps;    // hidden irreps staged
  std::map<int, int> x_st;    // irrep -> staged offset (floats)
  int xs = 0;                 // staged x floats per edge
  std::map<int, int> g_st;    // path -> staged offset of its grad_out block (backward)
  int gs = 0;                 // staged grad_out floats per receiver (backward)
};

std::string gen_producer(const Plan& P, const FwdConfig& F);
std::string gen_slice_helpers(const Plan& P, const FwdConfig& F, const std::vector<SliceLayout>& SL);
std::string gen_layout(const Plan& P, const FwdConfig& F, const std::vector<SliceLayout>& SL,
                       int extra_bytes, int& off_extra, int& smem_bytes);

cgtp_status upload_chat_tables(const Plan& P, const std::vector<SliceLayout>& SL, void** d_ent,
                               void** d_term, std::vector<int>& ent_begin);

}  // namespace cgtp
