// profile.h -- scoped event timing of library launches (see profile.cu).
#pragma once

#include <cuda_runtime.h>

namespace hsa {

// Brackets the launches issued inside the scope with events on stream s when profiling is on.
class ProfScope {
   public:
    ProfScope(const char *name, cudaStream_t s);
    ~ProfScope();
    ProfScope(const ProfScope &) = delete;
    ProfScope &operator=(const ProfScope &) = delete;

   private:
    int idx_;
    cudaStream_t s_;
};

}  // namespace hsa

#define HSA_PROF_CAT2(a, b) a##b
#define HSA_PROF_CAT(a, b) HSA_PROF_CAT2(a, b)
#define HSA_PROF(name, stream) ::hsa::ProfScope HSA_PROF_CAT(hsa_prof_, __LINE__)(name, stream)
