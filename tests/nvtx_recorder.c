/* nvtx_recorder.c -- test helper: an NVTX injection library that records
 * every range push (with its name) and pop into the file named by the
 * RKL_NVTX_LOG environment variable.  NVTX loads it when a process sets
 * NVTX_INJECTION64_PATH to the built .so; tests/test_nvtx.py builds it with
 * gcc and checks that each C-ABI entry point of librkl.so opens and closes a
 * range named after itself. */
#include <stdio.h>
#include <stdlib.h>

#include <nvtx3/nvToolsExt.h>

static FILE* g_log = NULL;

static int record_push(const char* name) {
  if (g_log) {
    fprintf(g_log, "push %s\n", name ? name : "");
    fflush(g_log);
  }
  return 0;
}

static int record_pop(void) {
  if (g_log) {
    fputs("pop\n", g_log);
    fflush(g_log);
  }
  return 0;
}

/* Called by NVTX on the first NVTX call of the process: replace the core
 * module's push-by-ASCII-name and pop entries with the recorders. */
int InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_export_table) {
  const NvtxExportTableCallbacks* cb = (const NvtxExportTableCallbacks*)get_export_table(NVTX_ETID_CALLBACKS);
  NvtxFunctionTable table = NULL;
  unsigned int size = 0;
  const char* path = getenv("RKL_NVTX_LOG");
  if (cb == NULL || path == NULL) return 0;
  if (!cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE, &table, &size) || size <= NVTX_CBID_CORE_RangePop) return 0;
  g_log = fopen(path, "w");
  if (g_log == NULL) return 0;
  *table[NVTX_CBID_CORE_RangePushA] = (NvtxFunctionPointer)record_push;
  *table[NVTX_CBID_CORE_RangePop] = (NvtxFunctionPointer)record_pop;
  return 1;
}
