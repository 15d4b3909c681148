/* NVTX injection library used by the tests: records every range push and pop that the process
 * makes, so a test can check the names and nesting of libmoba's NVTX ranges without a profiler.
 *
 * Loaded by NVTX itself when NVTX_INJECTION64_PATH names this file: NVTX calls
 * InitializeInjectionNvtx2 once, and this replaces the core module's RangePushA and RangePop
 * entries.  The log is one line per event ("+name" or "-") read back through
 * nvtx_recorder_log().  Build: gcc -shared -fPIC -I<cuda>/include nvtx_recorder.c */
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

static char g_log[1 << 16];
static size_t g_len;
static int g_depth;

static void append(const char* s) {
    size_t n = strlen(s);
    if (g_len + n + 1 >= sizeof(g_log)) return;
    memcpy(g_log + g_len, s, n);
    g_len += n;
    g_log[g_len] = '\0';
}

static int NVTX_API record_push(const char* message) {
    append("+");
    append(message ? message : "");
    append("\n");
    return g_depth++;
}

static int NVTX_API record_pop(void) {
    append("-\n");
    return --g_depth;
}

int NVTX_API InitializeInjectionNvtx2(NvtxGetExportTableFunc_t get_table) {
    const NvtxExportTableCallbacks* cb = (const NvtxExportTableCallbacks*)get_table(NVTX_ETID_CALLBACKS);
    NvtxFunctionTable table = NULL;
    unsigned int last = 0; /* highest valid index of the table */
    if (!cb || !cb->GetModuleFunctionTable(NVTX_CB_MODULE_CORE, &table, &last)) return 0;
    if (!table || last < NVTX_CBID_CORE_RangePop) return 0;
    *table[NVTX_CBID_CORE_RangePushA] = (NvtxFunctionPointer)record_push;
    *table[NVTX_CBID_CORE_RangePop] = (NvtxFunctionPointer)record_pop;
    return 1;
}

const char* nvtx_recorder_log(void) { return g_log; }
