/* A minimal NVTX injection library for the tracing test.
 *
 * NVTX v3 loads the library named by NVTX_INJECTION64_PATH on the first
 * NVTX call of a process and calls its InitializeInjectionNvtx2, which asks
 * for the callback export table and installs its own handlers in the CORE2
 * (domain) module's function table.  This one records domain creation,
 * range pushes and pops, one line each, in the file named by
 * CSA_NVTX_PROBE_LOG:
 *     domain <name>
 *     push <domain name> <message>
 *     pop <domain name>
 */
#include <nvtx3/nvToolsExt.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

struct probe_domain {
  char name[64];
};

static struct probe_domain g_domains[16];
static int g_n_domains = 0;

static void log_line(const char* kind, const char* a, const char* b) {
  const char* path = getenv("CSA_NVTX_PROBE_LOG");
  if (!path) return;
  FILE* f = fopen(path, "a");
  if (!f) return;
  if (b)
    fprintf(f, "%s %s %s\n", kind, a, b);
  else
    fprintf(f, "%s %s\n", kind, a);
  fclose(f);
}

static const char* domain_name(nvtxDomainHandle_t d) {
  return d ? ((const struct probe_domain*)d)->name : "(default)";
}

static nvtxDomainHandle_t NVTX_API probe_domain_create(const char* name) {
  if (g_n_domains >= 16) return NULL;
  struct probe_domain* d = &g_domains[g_n_domains++];
  strncpy(d->name, name ? name : "", sizeof(d->name) - 1);
  log_line("domain", d->name, NULL);
  return (nvtxDomainHandle_t)d;
}

static int NVTX_API probe_push(nvtxDomainHandle_t d, const nvtxEventAttributes_t* ev) {
  const char* msg = (ev && ev->messageType == NVTX_MESSAGE_TYPE_ASCII && ev->message.ascii)
                        ? ev->message.ascii
                        : "?";
  log_line("push", domain_name(d), msg);
  return 0;
}

static int NVTX_API probe_pop(nvtxDomainHandle_t d) {
  log_line("pop", domain_name(d), NULL);
  return 0;
}

int NVTX_API InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_table) {
  const NvtxExportTableCallbacks* cb =
      (const NvtxExportTableCallbacks*)get_table(NVTX_ETID_CALLBACKS);
  if (!cb || !cb->GetModuleFunctionTable) return 0;
  NvtxFunctionTable table = NULL;
  unsigned int size = 0;
  if (!cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE2, &table, &size) || !table) return 0;
  if (size > NVTX_CBID_CORE2_DomainCreateA)
    *table[NVTX_CBID_CORE2_DomainCreateA] = (NvtxFunctionPointer)probe_domain_create;
  if (size > NVTX_CBID_CORE2_DomainRangePushEx)
    *table[NVTX_CBID_CORE2_DomainRangePushEx] = (NvtxFunctionPointer)probe_push;
  if (size > NVTX_CBID_CORE2_DomainRangePop)
    *table[NVTX_CBID_CORE2_DomainRangePop] = (NvtxFunctionPointer)probe_pop;
  return 1;
}
