// Optional per-launch timing hook (moe_trace_attach): while attached, every
// kernel launch made by the entry points is bracketed by cudaEventRecord on
// its stream.  Events and the label / count storage belong to the caller.
#include "common.cuh"

namespace moe {
namespace trace {

namespace {
cudaEvent_t* g_events = nullptr;
const char** g_labels = nullptr;
int32_t g_capacity = 0;
int32_t* g_count = nullptr;
}  // namespace

void begin(const char* name, cudaStream_t s) {
  if (!g_events || *g_count >= g_capacity) return;
  cudaEventRecord(g_events[2 * *g_count], s);
  if (g_labels) g_labels[*g_count] = name;
}

void end(cudaStream_t s) {
  if (!g_events || *g_count >= g_capacity) return;
  cudaEventRecord(g_events[2 * *g_count + 1], s);
  ++*g_count;
}

}  // namespace trace
}  // namespace moe

extern "C" {

moe_status moe_trace_attach(void* const* events, int32_t capacity, const char** labels, int32_t* count) {
  if (!events || capacity <= 0 || !count) return MOE_ERR_INVALID_ARG;
  moe::trace::g_events = (cudaEvent_t*)events;
  moe::trace::g_labels = labels;
  moe::trace::g_capacity = capacity;
  moe::trace::g_count = count;
  *count = 0;
  return MOE_OK;
}

moe_status moe_trace_detach(void) {
  moe::trace::g_events = nullptr;
  moe::trace::g_labels = nullptr;
  moe::trace::g_capacity = 0;
  moe::trace::g_count = nullptr;
  return MOE_OK;
}

}  // extern "C"
