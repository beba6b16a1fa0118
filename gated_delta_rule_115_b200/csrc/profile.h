// profile.h -- launch bracketing for the opt-in kernel timing (muir_profile.h).
#pragma once

#include <cuda_runtime.h>

namespace muir {
namespace prof {

bool enabled();
// Records a start event on st; returns a ticket (-1 when profiling is off).
int begin(const char* name, cudaStream_t st);
// Records the matching stop event.
void end(int ticket, cudaStream_t st);

struct Scope {
    int ticket;
    cudaStream_t st;
    Scope(const char* name, cudaStream_t s) : ticket(enabled() ? begin(name, s) : -1), st(s) {}
    ~Scope() { if (ticket >= 0) end(ticket, st); }
};

}  // namespace prof
}  // namespace muir

// Launch a kernel inside a timing scope: MUIR_TIMED("name", stream, kernel<<<...>>>(...));
#define MUIR_TIMED(name, st, ...)              \
    do {                                       \
        ::muir::prof::Scope muir_scope_(name, st); \
        __VA_ARGS__;                           \
    } while (0)
