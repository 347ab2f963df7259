// Per-shape choice between the dense and the 2:4 GEMM of one weight.
//
// [P2] "Ask which sparse implementations were actually selected": a layer whose weights meet
// the 2:4 pattern is only eligible for the sparse path; whether the sparse implementation is
// selected is a separate, per-problem-size decision, and dense may win at some sizes.  Here:
//   * sp24_gemm_select times both GEMMs of a shape on the caller's stream (CUDA events around
//     `reps` back-to-back launches after one warm-up launch each) and records the faster one
//     for (device, x format, weight format, M, N, K);
//   * sp24_gemm_choice answers from that record, else from a rule of measured crossovers on
//     B200 (the repository's benchmark at N = K = 5120): 16-bit weights go 2:4 from M = 128
//     (the CTA-pair tensor-core kernels: 1.10x at M = 128, 1.18-1.49x from M = 1024; 0.97-1.01x
//     at M = 1 and 16); NVFP4 weights with 16-bit activations go 2:4 from M = 128 (1.34-1.61x),
//     below it the dense decode and skinny kernels win (0.87-0.92x, and dense 47 against 50 us
//     at M = 80); NVFP4 weights with NVFP4 activations stay dense (the dense FP4 MMA against
//     the 16-bit sparse MMA: 0.45-0.49x, 1.05x only at M = 16); weights of fewer than 2^20
//     entries stay dense (launch-bound: 5.1 vs 5.6 us for a [256, 512] weight at M = 16, the
//     dense kernel starts sooner);
//   * sp24_gemm_auto runs the chosen GEMM (asynchronous; usable under graph capture).
// Host code only: the GEMMs are the library's own entry points.
#include "sp24_internal.cuh"

#include <map>
#include <mutex>
#include <tuple>

namespace sp24 {
namespace {

using Key = std::tuple<int, int, int, int64_t, int64_t, int64_t>;  // device, x fmt, w fmt, M, N, K

std::mutex g_sel_mu;
std::map<Key, int>& sel_table() {
  static std::map<Key, int> t;
  return t;
}

bool is16(int f) { return f == SP24_F16 || f == SP24_BF16; }

// The measured-crossover rule (see the file comment).  -1: no 2:4 path for these formats.
int rule_choice(int x_format, int w_format, int64_t M, int64_t N, int64_t K) {
  const bool pair16 = is16(x_format) && is16(w_format), w4a16 = is16(x_format) && w_format == SP24_NVFP4;
  if (!pair16 && !w4a16 && !(x_format == SP24_NVFP4 && w_format == SP24_NVFP4)) return -1;
  if (N * K < (int64_t)1 << 20) return 0;  // launch-bound: the dense kernel starts sooner
  if (pair16 || w4a16) return M >= 128 ? 1 : 0;
  return 0;
}

int device_now() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) d = -1;
  return d;
}

}  // namespace
}  // namespace sp24

using namespace sp24;

extern "C" int sp24_gemm_choice(int x_format, int w_format, int64_t M, int64_t N, int64_t K, int* use_sparse,
                                int* measured) {
  if (!use_sparse) return SP24_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0) return SP24_ERR_SHAPE;
  const int rule = rule_choice(x_format, w_format, M, N, K);
  if (rule < 0) return SP24_ERR_DTYPE;
  {
    std::lock_guard<std::mutex> lk(g_sel_mu);
    auto it = sel_table().find(Key(device_now(), x_format, w_format, M, N, K));
    if (it != sel_table().end()) {
      *use_sparse = it->second;
      if (measured) *measured = 1;
      return SP24_OK;
    }
  }
  *use_sparse = rule;
  if (measured) *measured = 0;
  return SP24_OK;
}

extern "C" int sp24_gemm_choice_reset(void) {
  std::lock_guard<std::mutex> lk(g_sel_mu);
  sel_table().clear();
  return SP24_OK;
}

extern "C" int sp24_gemm_select(const sp24_operand* x, const sp24_operand* w_dense, const sp24_sparse_operand* w_sparse,
                                int64_t M, int64_t N, int64_t K, float* y, void* workspace, int64_t workspace_bytes,
                                int reps, int* use_sparse, float* us_dense, float* us_sparse, void* stream) {
  if (!x || !w_dense || !w_sparse || !use_sparse || reps < 1) return SP24_ERR_INVALID_ARG;
  if (w_dense->format != w_sparse->format) return SP24_ERR_DTYPE;
  if (rule_choice(x->format, w_dense->format, M, N, K) < 0) return SP24_ERR_DTYPE;
  cudaStream_t s = as_stream(stream);
  cudaEvent_t ev[4];
  for (auto& e : ev)
    if (cudaEventCreate(&e) != cudaSuccess) return SP24_ERR_CUDA;
  float ms[2] = {0.0f, 0.0f};
  int st = SP24_OK;
  for (int which = 0; which < 2 && st == SP24_OK; ++which) {
    auto run = [&]() {
      return which ? sp24_gemm_sparse24(x, w_sparse, M, N, K, y, workspace, workspace_bytes, 0, stream)
                   : sp24_gemm_dense(x, w_dense, M, N, K, y, workspace, workspace_bytes, 0, stream);
    };
    st = run();  // warm-up (and the first error, if any)
    if (st) break;
    if (cudaEventRecord(ev[2 * which], s) != cudaSuccess) st = SP24_ERR_CUDA;
    for (int r = 0; r < reps && st == SP24_OK; ++r) st = run();
    if (st == SP24_OK && cudaEventRecord(ev[2 * which + 1], s) != cudaSuccess) st = SP24_ERR_CUDA;
  }
  if (st == SP24_OK && cudaEventSynchronize(ev[3]) != cudaSuccess) st = SP24_ERR_CUDA;
  if (st == SP24_OK && (cudaEventElapsedTime(&ms[0], ev[0], ev[1]) != cudaSuccess ||
                        cudaEventElapsedTime(&ms[1], ev[2], ev[3]) != cudaSuccess))
    st = SP24_ERR_CUDA;
  for (auto& e : ev) cudaEventDestroy(e);
  if (st) return st;
  const int choice = ms[1] < ms[0] ? 1 : 0;
  *use_sparse = choice;
  if (us_dense) *us_dense = 1000.0f * ms[0] / reps;
  if (us_sparse) *us_sparse = 1000.0f * ms[1] / reps;
  std::lock_guard<std::mutex> lk(g_sel_mu);
  sel_table()[Key(device_now(), x->format, w_dense->format, M, N, K)] = choice;
  return SP24_OK;
}

extern "C" int sp24_gemm_auto(const sp24_operand* x, const sp24_operand* w_dense, const sp24_sparse_operand* w_sparse,
                              int64_t M, int64_t N, int64_t K, float* y, void* workspace, int64_t workspace_bytes,
                              int* used_sparse, void* stream) {
  if (!x || !w_dense || !w_sparse) return SP24_ERR_INVALID_ARG;
  if (w_dense->format != w_sparse->format) return SP24_ERR_DTYPE;
  int choice = 0;
  const int st = sp24_gemm_choice(x->format, w_dense->format, M, N, K, &choice, nullptr);
  if (st) return st;
  if (used_sparse) *used_sparse = choice;
  return choice ? sp24_gemm_sparse24(x, w_sparse, M, N, K, y, workspace, workspace_bytes, 0, stream)
                : sp24_gemm_dense(x, w_dense, M, N, K, y, workspace, workspace_bytes, 0, stream);
}
