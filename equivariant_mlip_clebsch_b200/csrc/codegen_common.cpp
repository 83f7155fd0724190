// codegen_common.cpp -- device prelude text and the Chat build tables.
#include "codegen_common.hpp"

#include <cstring>

namespace cgtp {

const char* kPrelude =
#include "device_prelude.inc"
    ;

// One entry per Chat element that some role reads: (dst offset inside the
// edge's Chat block, first term, number of terms); one term per non-zero
// C_p[m1][m2][m3]: (column l2^2+m2 of Y, coefficient as FP32 bits).
cgtp_status upload_chat_tables(const Plan& P, const std::vector<SliceLayout>& SL, void** d_ent,
                               void** d_term, std::vector<int>& ent_begin) {
  std::vector<int> ent, term;
  ent_begin.assign(1, 0);
  for (const SliceLayout& sl : SL) {
    for (int pi : sl.paths) {
      const Path& p = P.paths[pi];
      const int n1 = 2 * p.l1 + 1, n2 = 2 * p.l2 + 1, n3 = 2 * p.l3 + 1;
      const double* C = P.coeff.data() + p.c_off;
      for (int m3 = 0; m3 < n3; ++m3)
        for (int m1 = 0; m1 < n1; ++m1) {
          const int tb = (int)term.size() / 2;
          int cnt = 0;
          for (int m2 = 0; m2 < n2; ++m2) {
            const double c = C[((size_t)m1 * n2 + m2) * n3 + m3];
            if (c == 0.0) continue;
            const float cf = (float)c;
            int bits;
            std::memcpy(&bits, &cf, 4);
            term.push_back(p.l2 * p.l2 + m2);
            term.push_back(bits);
            ++cnt;
          }
          ent.push_back(sl.ch_off.at(pi) + chat_pos(p.l1, p.l3, m1, m3));
          ent.push_back(tb);
          ent.push_back(cnt);
          ent.push_back(0);
        }
    }
    ent_begin.push_back((int)ent.size() / 4);
  }
  if (P.host_only) return CGTP_OK;
  if (ent.empty()) ent.assign(4, 0);
  if (term.empty()) term.assign(2, 0);
  if (cudaMalloc(d_ent, ent.size() * sizeof(int)) != cudaSuccess ||
      cudaMalloc(d_term, term.size() * sizeof(int)) != cudaSuccess)
    return fail(CGTP_ERR_OOM, "cudaMalloc of the Chat tables");
  CGTP_CUDA_TRY(cudaMemcpy(*d_ent, ent.data(), ent.size() * sizeof(int), cudaMemcpyHostToDevice));
  CGTP_CUDA_TRY(cudaMemcpy(*d_term, term.data(), term.size() * sizeof(int), cudaMemcpyHostToDevice));
  return CGTP_OK;
}

}  // namespace cgtp
