/* A minimal NVTX tool for the tests: loaded by NVTX through
 * NVTX_INJECTION64_PATH, it writes every range push, pop and mark of the
 * domain API to the file named by ZERO_NVTX_LOG, one line each:
 *   domain <name> / push <message> / pop / mark <message>
 * It implements only the documented injection entry point of NVTX v3
 * (InitializeInjectionNvtx2, which receives the export-table getter) and
 * fills in the domain callbacks the library uses. */
#define NVTX_NO_IMPL
#include <nvtx3/nvToolsExt.h>

#include <stdio.h>
#include <stdlib.h>

static FILE *g_log;

static void put(const char *what, const nvtxEventAttributes_t *a) {
    if (!g_log) return;
    const char *msg = (a && a->messageType == NVTX_MESSAGE_TYPE_ASCII) ? a->message.ascii : "?";
    fprintf(g_log, "%s %s\n", what, msg);
    fflush(g_log);
}

static nvtxDomainHandle_t NVTX_API on_domain_create(const char *name) {
    static int handle;
    if (g_log) {
        fprintf(g_log, "domain %s\n", name);
        fflush(g_log);
    }
    return (nvtxDomainHandle_t)&handle;
}

static int NVTX_API on_push(nvtxDomainHandle_t d, const nvtxEventAttributes_t *a) {
    (void)d;
    put("push", a);
    return 0;
}

static int NVTX_API on_pop(nvtxDomainHandle_t d) {
    (void)d;
    if (g_log) {
        fprintf(g_log, "pop\n");
        fflush(g_log);
    }
    return 0;
}

static void NVTX_API on_mark(nvtxDomainHandle_t d, const nvtxEventAttributes_t *a) {
    (void)d;
    put("mark", a);
}

__attribute__((visibility("default"))) int NVTX_API InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get) {
    const NvtxExportTableCallbacks *cb = (const NvtxExportTableCallbacks *)get(NVTX_ETID_CALLBACKS);
    NvtxFunctionTable table = 0;
    unsigned int size = 0;
    if (!cb || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE2, &table, &size) || !table)
        return 0;
    if (size <= NVTX_CBID_CORE2_DomainCreateA) return 0;
    *table[NVTX_CBID_CORE2_DomainCreateA] = (NvtxFunctionPointer)on_domain_create;
    *table[NVTX_CBID_CORE2_DomainRangePushEx] = (NvtxFunctionPointer)on_push;
    *table[NVTX_CBID_CORE2_DomainRangePop] = (NvtxFunctionPointer)on_pop;
    *table[NVTX_CBID_CORE2_DomainMarkEx] = (NvtxFunctionPointer)on_mark;
    const char *path = getenv("ZERO_NVTX_LOG");
    g_log = path ? fopen(path, "w") : NULL;
    return 1;
}
