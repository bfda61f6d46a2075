/*
 * probe_rows.h -- measurement helper of the benchmark (libsdm_probe.so), not
 * part of the SDM C ABI in include/sdm.h.
 *
 * sdm_probe_random_rows launches `ctas` CTAs of 256 threads that each move, per
 * iteration, rows_in_flight (4 or 8) random whole rows of 64 floats (256
 * bytes) per group of 8 threads in `table` (nrows rows, device memory, 16-byte
 * aligned): loads only (rmw = 0) or load, add and store back (rmw = 1), `iters`
 * times.  Bytes moved = ctas * 32 * rows_in_flight * iters * 256 (times 2 with
 * rmw).  It gives the HBM ceiling of the recurrence's random-row access
 * pattern.  Asynchronous on `stream` (a cudaStream_t); the table is modified
 * when rmw = 1.  Returns one of the codes below.
 */
#ifndef SDM_PROBE_ROWS_H_
#define SDM_PROBE_ROWS_H_

#if defined(__GNUC__)
#define SDM_PROBE_API __attribute__((visibility("default")))
#else
#define SDM_PROBE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  SDM_PROBE_OK = 0,
  SDM_PROBE_ERR_NULL = 1,        /* table is NULL */
  SDM_PROBE_ERR_DIMS = 2,        /* nrows, ctas or iters out of range */
  SDM_PROBE_ERR_ALIGN = 3,       /* table not 16-byte aligned */
  SDM_PROBE_ERR_UNSUPPORTED = 5, /* rows_in_flight other than 4 or 8 */
  SDM_PROBE_ERR_CUDA = 6         /* the launch failed */
};

SDM_PROBE_API int sdm_probe_random_rows(float* table, long long nrows, int rmw,
                                        int rows_in_flight, int ctas, int iters, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SDM_PROBE_ROWS_H_ */
