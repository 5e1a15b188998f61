// debug_check.cuh -- index checks of the debug build.
//
// Built with -DCSA_DEBUG, the kernels check the shared-memory, tensor-memory,
// score-buffer, candidate-list and output indices they compute against the
// bounds of what they address.  A failed check records itself in the device
// error word (code kErrDebugCheck, where, the index, the bound; the first
// failure wins) and the access is skipped: nothing traps, the kernel runs
// on, and csa_last_device_error() reports CSA_ERR_DEBUG_CHECK.  In the
// release build CSA_CHECK_INDEX is the constant `true` and costs nothing.
//
// The recording function is plain C++ on the host (no CUDA), so the host can
// exercise exactly the code that records a failure.
#pragma once
#include <cstdint>

#if defined(__CUDACC__)
#define CSA_HD __host__ __device__
#else
#define CSA_HD
#endif

namespace csa {

enum : int { kErrDebugCheck = 6 };

// Where a debug check sits (the error word's second entry).
enum CheckSite : int {
    kChkKeyStage = 1,    // producer: key tile destination in shared memory
    kChkQueryBlock = 2,  // producer: query block destination in shared memory
    kChkTmemMma = 3,     // MMA: accumulator columns of a tile
    kChkTmemEpi = 4,     // epilogue: accumulator columns it loads
    kChkScoreBuf = 5,    // epilogue: key slot in the CTA's score buffer
    kChkListPos = 6,     // selector: candidate list position
    kChkSelOut = 7,      // select kernel: staging slot in shared memory
    kChkOutSlot = 8      // select kernel: output slot of a query row
};

// Records a failed check (index not in [0, bound)) in `word` unless an
// earlier failure is recorded there; returns whether the index is in bounds.
CSA_HD inline bool record_check(int *word, int site, long long index, long long bound)
{
    if (index >= 0 && index < bound)
        return true;
#if defined(__CUDA_ARCH__)
    if (atomicCAS(&word[0], 0, kErrDebugCheck) == 0) {
#else
    if (word[0] == 0) {
        word[0] = kErrDebugCheck;
#endif
        word[1] = site;
        word[2] = static_cast<int>(index);
        word[3] = static_cast<int>(bound);
    }
    return false;
}

} // namespace csa

#if defined(CSA_DEBUG) && defined(__CUDA_ARCH__)
// Needs g_csa_error (ptx.cuh) in scope.
#define CSA_CHECK_INDEX(site, index, bound) \
    (::csa::record_check(::csa::g_csa_error, (site), static_cast<long long>(index), \
                         static_cast<long long>(bound)))
#else
#define CSA_CHECK_INDEX(site, index, bound) true
#endif
