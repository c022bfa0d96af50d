// prof.h -- kernel identifiers and the launch-timing scope used around every launch.
#pragma once

#include <cuda_runtime.h>

namespace dynconv {

enum KernelId {
    kSimtGen = 0, kSimtWiden, kSimtConvFwd, kSimtConvBwd, kSimtDB, kSimtHTX, kSimtDh,
    kCheckSeqlens, kTcGen, kTcLowrankFwd, kTcLowrankBwd, kTcGenBwd, kTcReduce,
    kTcHeadwiseFwd, kTcHeadwiseBwd, kTcPrep, kDecodeGen, kDecodeConv, kSimtRope,
    kKernelCount
};

// Records an event on `st` at construction and another at destruction when
// profiling is enabled; wrap exactly one kernel launch in it.
class ProfScope {
  public:
    ProfScope(int id, cudaStream_t st);
    ~ProfScope();
    ProfScope(const ProfScope&) = delete;
    ProfScope& operator=(const ProfScope&) = delete;

  private:
    int id_;
    cudaStream_t st_;
    cudaEvent_t a_;
};

const char* kernel_name(int id);

}  // namespace dynconv

#define DC_LAUNCH(id, st, ...)                      \
    do {                                            \
        ::dynconv::ProfScope _dc_scope((id), (st)); \
        __VA_ARGS__;                                \
    } while (0)
