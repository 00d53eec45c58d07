/* sa_trace.h -- phase-timeline hook of the traced build of the library.
 *
 * paged_kv_cache_sa_b200/build.py --trace compiles the same sources with -DSA_TRACE into
 * lib/libsa_trace.so, which exports everything libsa.so exports plus sa_trace_set; the
 * kernels then store %globaltimer (ns) at fixed points into the installed buffer:
 *   buf[kernel][cta][event], kernel 0..4 (scoring, selection, attention, merge, the
 *   single-launch decode's phase boundaries), cta < 1024 (blockIdx.x + blockIdx.y *
 *   gridDim.x), event < 16; the event numbers are listed in
 *   paged_kv_cache_sa_b200/timeline.py.  Slots that no CTA reaches keep their value.
 * libsa.so has no trace points and does not export this call.
 */
#ifndef SA_TRACE_H
#define SA_TRACE_H

#ifdef __cplusplus
extern "C" {
#endif

/* Install the device buffer (5 * 1024 * 16 uint64, caller-owned) for the kernels of the
 * calls that follow; NULL stops recording.  Returns SA_OK. */
int sa_trace_set(void* device_buf);

#ifdef __cplusplus
}
#endif

#endif
