/*
 * muir_profile.h -- opt-in per-kernel timing of libmuir launches.
 *
 * Not part of the recurrence; the pages have no counterpart.  When enabled,
 * every kernel libmuir launches is bracketed by two CUDA events recorded on
 * the launch stream.  muir_profile_collect() waits for the recorded events
 * (host synchronisation on them), adds each elapsed time to a per-kernel
 * total and recycles the events.  Totals persist until muir_profile_reset().
 * Thread safety: all functions take an internal lock.
 */
#ifndef MUIR_PROFILE_H_
#define MUIR_PROFILE_H_

#ifdef __cplusplus
extern "C" {
#endif

/* on != 0 starts recording events around launches; 0 stops (pending events stay). */
void muir_profile_enable(int on);
/* Clears all totals and pending events. */
void muir_profile_reset(void);
/* Waits for pending events and accumulates them; returns 0, or a cudaError_t value. */
int muir_profile_collect(void);
/* Number of distinct kernel names seen so far. */
int muir_profile_count(void);
/* Name of kernel i (static storage until the next reset), NULL if out of range. */
const char* muir_profile_name(int i);
/* Total milliseconds and launch count of kernel i since the last reset. */
double muir_profile_total_ms(int i);
long long muir_profile_launches(int i);

#ifdef __cplusplus
}
#endif

#endif /* MUIR_PROFILE_H_ */
