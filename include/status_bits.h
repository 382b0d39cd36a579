/* Device status bits written by the kernels into the first word of a workspace or plan
 * (read with bsa_get_status).  Shared by the C ABI header and the device code. */
#ifndef SELECTED_ATTENTION_STATUS_BITS_H_
#define SELECTED_ATTENTION_STATUS_BITS_H_
#define SA_DEV_BAD_INDEX 1u  /* a selected block id at or past the sequence's block count (dropped) */
#define SA_DEV_BAD_SEQLEN 2u /* cu_seqlens not non-decreasing, or its last entry != T (units skipped) */
#define SA_DEV_TIMEOUT 4u    /* a kernel wait exceeded its limit; the kernel stopped early */
#endif
