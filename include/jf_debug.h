/* jf_debug.h -- test hooks of the debug build of libjf (libjf_debug.so, built with JF_DEBUG).
 *
 * The pages describe no such calls; they exist to test the library's failure detection without faulting a GPU.
 * In the debug build every bounded device wait gives up after 50 ms (2 s in the release build).
 */
#ifndef JF_DEBUG_H_
#define JF_DEBUG_H_

#include "jf.h"

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------------------------------
 * jf_debug_hold -- makes jf_tree_attention's wait run out.
 *
 * With on != 0, every CTA of the attention kernel of later jf_tree_attention / jf_tree_attention_fp8 calls
 * first waits for the hold to be released; nothing releases it during a call, so the wait gives up after
 * the debug build's 50 ms limit, before any copy or MMA is issued: the call writes JF_ERR_TIMEOUT to
 * dev_status, leaves out unwritten and returns, and the context stays usable.  on = 0 releases the hold.
 * Returns JF_ERR_CUDA if the device flag cannot be written.  Device-wide: set it only between calls.
 * ------------------------------------------------------------------------------------------ */
JF_API jf_status jf_debug_hold(int on);

#ifdef __cplusplus
}
#endif

#endif  /* JF_DEBUG_H_ */
