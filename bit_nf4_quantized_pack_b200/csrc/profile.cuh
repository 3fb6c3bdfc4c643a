// Internal launch-timing scope (see profile.cu and qlora_profile_* in the
// public header).
#pragma once

#include <cuda_runtime.h>

namespace qnf4 {

// Kernel classes, matching QLORA_PROF_* in qlora_nf4.h.
enum ProfKind {
  kProfFusedFwd = 0,
  kProfFusedBwd = 1,
  kProfSkinny = 2,
  kProfQuantize = 3,
  kProfDequantize = 4,
  kProfGemv = 5,
  kProfOther = 6,
  kProfKinds = 7
};

// Counts one launch of kind `id` and, while profiling is enabled, brackets it
// with CUDA events on stream `s` (constructed right before the launch,
// destroyed right after it).
class ProfScope {
 public:
  ProfScope(int id, cudaStream_t s);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;

 private:
  int id_;
  cudaStream_t s_;
  void* a_;
};

void prof_count_only(int id);

// True while launches of kind `id` are being timed.  The backward then runs
// its rank-r launches in order on the caller's stream instead of beside dX,
// so that each class's events bracket that class's work alone.
bool prof_timing(int id);

}  // namespace qnf4
