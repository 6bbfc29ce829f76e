/*
 * dg_noalloc.h -- the canvas update of dg.h without a caller-provided workspace.
 *
 * The pages that define the method have no counterpart to this call: it is a
 * deployment convenience, computing exactly what dg_canvas_update computes.
 *
 * Who needs it: a caller that cannot hand the library any device scratch -- for
 * instance a sampling step embedded in another engine that owns every byte of device
 * memory and offers none to its plug-ins, or a loop that must not call cudaMalloc /
 * cudaFree once it runs (cudaFree waits for the whole device, which would stall the
 * caller's other streams).  This entry point neither allocates nor frees device memory
 * and calls no allocating library; its scratch is a fixed array compiled into libdg.
 */
#ifndef DG_NOALLOC_H
#define DG_NOALLOC_H

#include "dg.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Same arguments, result and validation as dg_canvas_update, minus the workspace.
 *
 * Scratch: one fixed device array of 2048 (row, slice) partial-reduction records
 * (16 bytes each, 32 KB) per CUDA context that loads libdg's device image, shared by
 * every call in that context.  The call needs C x s records, s the number of
 * vocabulary slices the update uses (s = ceil(592 / C), at most ceil(V / 4096)), which
 * is below 592 + C <= 1616 for every C <= 1024; a shape needing more than 2048 is
 * rejected with DG_ERR_CAPACITY before anything is launched.
 *
 * After a call the array holds that call's per-(row, slice) max, sum of exp(l - max)
 * and first argmax of the logits; nothing reads it afterwards.
 *
 * Concurrency: two calls in the same context that may run at the same time (different
 * streams without an ordering between them, or several host threads) write the same
 * array and race.  Order them, e.g. on one stream.
 *
 * Set-up: the array's device address differs per CUDA context, so the first call in
 * each context (the primary context of a device, or a context the caller created and
 * made current) looks it up with cudaGetSymbolAddress, with that context current, and
 * caches it under the context's unique id (cuCtxGetId; ids are never reused within a
 * process, so a context destroyed by cudaDeviceReset and its successor never share an
 * entry).  Make that first call before any stream capture begins.  Errors:
 * DG_ERR_INVALID_ARG as dg_canvas_update; DG_ERR_CAPACITY as above; DG_ERR_CUDA if
 * there is no current context, or the look-up or a launch fails. */
dg_status dg_canvas_update_noalloc(const float* d_logits, int32_t C, int32_t V, int32_t n_renoise, uint64_t seed,
                                   uint32_t step, int32_t* d_canvas, float* d_conf, dg_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* DG_NOALLOC_H */
