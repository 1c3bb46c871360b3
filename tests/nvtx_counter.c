/* An NVTX tool for the tests (loaded through NVTX_INJECTION64_PATH): it
 * replaces the range push and pop callbacks with counters, keeps the pushed
 * names, and at exit writes them to the file named by NVTX_COUNTER_OUT. */
#include <nvtx3/nvToolsExt.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static int pushes, pops;
static char names[8192];

static int count_push(const char* name) {
  ++pushes;
  if (strlen(names) + strlen(name) + 2 < sizeof names) {
    strcat(names, name);
    strcat(names, "\n");
  }
  return 0;
}

static int count_pop(void) {
  ++pops;
  return 0;
}

static void report(void) {
  const char* path = getenv("NVTX_COUNTER_OUT");
  FILE* f = path ? fopen(path, "w") : NULL;
  if (!f) return;
  fprintf(f, "pushes %d\npops %d\n%s", pushes, pops, names);
  fclose(f);
}

int InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_table) {
  const NvtxExportTableCallbacks* cb = (const NvtxExportTableCallbacks*)get_table(NVTX_ETID_CALLBACKS);
  NvtxFunctionTable table = NULL;
  unsigned int size = 0;
  if (!cb || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE, &table, &size) || !table) return 0;
  if (size > NVTX_CBID_CORE_RangePushA) *table[NVTX_CBID_CORE_RangePushA] = (NvtxFunctionPointer)count_push;
  if (size > NVTX_CBID_CORE_RangePop) *table[NVTX_CBID_CORE_RangePop] = (NvtxFunctionPointer)count_pop;
  atexit(report);
  return 1;
}
