// msda_api_util.h -- argument checks and launch-status helpers shared by the
// C entry points (msda_api.cpp, msda_api_tiled.cpp).  Not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "msda.h"
#include "msda_internal.h"

namespace msda {
namespace api {

constexpr int64_t kI32Max = 2147483647LL;
constexpr int64_t kGuard = (int64_t)1 << 62;

// The cudaError_t behind the calling thread's last MSDA_ERR_CUDA.
extern thread_local int g_last_cuda_error;

struct Span {
    const void *p;
    int64_t bytes;
};

// Validated problem: element counts and launch-side metadata.
struct Problem {
    int64_t items;    // N*Lq*M
    int64_t samples;  // N*Lq*M*L*K: per-head tensors (weights, logits)
    int64_t lsamples; // N*Lq*G*L*K: per-group tensors (locations, offsets)
    int64_t n_value;  // N*S*M*D
    int64_t n_out;    // N*Lq*M*D
    int esz;          // value element size
    int nchunks;      // 16-byte chunks per value row
    int lanes;        // lanes per row: next power of two >= nchunks, at most 32
    Levels lv;
};

// a * b with a, b >= 0; false if the product exceeds `limit`.
bool mul_le(int64_t a, int64_t b, int64_t limit, int64_t *out);
bool aligned(const void *p, uintptr_t a);
bool overlap(Span a, Span b);
// True if any output overlaps any input or another output.
bool any_alias(const Span *outs, int nout, const Span *ins, int nin);
// Dims, level metadata and size limits (no pointers).
msda_status check_dims(msda_dtype dt, const int64_t *shapes, const int64_t *starts,
                       const msda_dims &d, Problem *pr);
// Deformable groups: G groups of M/G consecutive heads share one set of
// sampling locations (G = M: every head has its own).
msda_status check_groups(const msda_dims &d, int64_t G, Problem *pr);
msda_status cuda_status(cudaError_t e);
// Status of a launch.  The bounds-checked build also waits for the stream,
// reads the device word, and clears it if the kernel recorded a violation.
msda_status launched(cudaError_t e, cudaStream_t s);

#ifdef MSDA_CHECKED
extern std::atomic<int64_t> g_check_limit;
extern thread_local int64_t g_violation_count;
extern thread_local int64_t g_violation_first;
#endif

template <class Params>
void set_dims(Params *p, const msda_dims &d, int64_t G, const Problem &pr)
{
    p->items = pr.items;
    p->Lq = (int)d.Lq;
    p->S = (int)d.S;
    p->M = (int)d.M;
    p->D = (int)d.D;
    p->L = (int)d.L;
    p->K = (int)d.K;
    p->G = (int)G;
    p->Hg = (int)(d.M / G);
    // item indices N*Lq*M stay below 2^31 (check_dims), so the kernels
    // divide them in 32 bits
    p->dM = msda::make_fastdiv((unsigned)(d.M > 0 ? d.M : 1));
    p->dLq = msda::make_fastdiv((unsigned)(d.Lq > 0 ? d.Lq : 1));
    p->dHg = msda::make_fastdiv((unsigned)(p->Hg > 0 ? p->Hg : 1));
    p->nchunks = pr.nchunks;
    p->lv = pr.lv;
}

// The bounds-check fields of a launch: the value map's element count (or the
// lowered test limit) and the device word.  Nothing in the default build.
template <class Params>
msda_status set_checks(Params *p, const Problem &pr)
{
    p->check_limit = pr.n_value;
    p->check = nullptr;
#ifdef MSDA_CHECKED
    const int64_t lim = g_check_limit.load();
    if (lim >= 0 && lim < p->check_limit) p->check_limit = lim;
    p->check = msda::check_word();
    if (!p->check) {
        const cudaError_t e = cudaGetLastError();
        return cuda_status(e != cudaSuccess ? e : cudaErrorUnknown);
    }
#endif
    return MSDA_OK;
}

}  // namespace api
}  // namespace msda
