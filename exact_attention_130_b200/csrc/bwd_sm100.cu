// bwd_sm100.cu -- attention backward (placeholder until the kernel lands).
#include "fa_internal.h"

namespace fa {

namespace {
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
}  // namespace

size_t bwd_workspace_bytes(int B, int H, int N, int d) {
  const size_t rows = size_t(B) * H * N;
  return align256(rows * d * 4) + align256(rows * 4);
}

fa_status launch_bwd(const void*, const void*, const void*, const void*, const float*,
                     const void*, void*, void*, void*, int, int, int, int, float, bool, void*,
                     const LaunchCtx&) {
  set_last_error("fa_bwd: not built yet");
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
