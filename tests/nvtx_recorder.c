/* A minimal NVTX tool for the tests: loaded by the NVTX v3 headers of a
 * program when NVTX_INJECTION64_PATH names this library.  It subscribes to
 * the domain calls (create, push, pop) of the "core v2" callback module and
 * writes one line per call to the file NVTX_RECORD_FILE names:
 *   domain <name>
 *   push <domain> <message>
 *   pop <domain>
 * Build: gcc -shared -fPIC -I<cuda>/include nvtx_recorder.c -o librec.so
 * Test infrastructure only; the library never links it. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#define MAX_DOMAINS 16

static FILE* g_out;
static char g_names[MAX_DOMAINS][64];
static int g_n;

/* a domain handle is 1 + its index, as an opaque pointer */
static const char* domain_name(nvtxDomainHandle_t d) {
  const size_t i = (size_t)d;
  return i >= 1 && i <= (size_t)g_n ? g_names[i - 1] : "(default)";
}

static nvtxDomainHandle_t NVTX_API rec_create(const char* name) {
  if (g_n == MAX_DOMAINS) return (nvtxDomainHandle_t)0;
  snprintf(g_names[g_n], sizeof g_names[0], "%s", name ? name : "");
  ++g_n;
  fprintf(g_out, "domain %s\n", g_names[g_n - 1]);
  fflush(g_out);
  return (nvtxDomainHandle_t)(size_t)g_n;
}

static int NVTX_API rec_push(nvtxDomainHandle_t d, const nvtxEventAttributes_t* a) {
  const char* msg = a && a->messageType == NVTX_MESSAGE_TYPE_ASCII ? a->message.ascii : "?";
  fprintf(g_out, "push %s %s\n", domain_name(d), msg);
  fflush(g_out);
  return 0;
}

static int NVTX_API rec_pop(nvtxDomainHandle_t d) {
  fprintf(g_out, "pop %s\n", domain_name(d));
  fflush(g_out);
  return 0;
}

int NVTX_API InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_table) {
  const char* path = getenv("NVTX_RECORD_FILE");
  const NvtxExportTableCallbacks* cb;
  NvtxFunctionTable table = 0;
  unsigned int size = 0;
  if (!path || !get_table) return 0;
  cb = (const NvtxExportTableCallbacks*)get_table(NVTX_ETID_CALLBACKS);
  if (!cb || !cb->GetModuleFunctionTable || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE2, &table, &size))
    return 0;
  if (size <= NVTX_CBID_CORE2_DomainCreateA) return 0;
  g_out = fopen(path, "w");
  if (!g_out) return 0;
  *table[NVTX_CBID_CORE2_DomainCreateA] = (NvtxFunctionPointer)rec_create;
  *table[NVTX_CBID_CORE2_DomainRangePushEx] = (NvtxFunctionPointer)rec_push;
  *table[NVTX_CBID_CORE2_DomainRangePop] = (NvtxFunctionPointer)rec_pop;
  return 1;
}
