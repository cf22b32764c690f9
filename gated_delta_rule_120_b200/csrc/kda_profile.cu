// kda_profile.cu — optional per-kernel event timing of the library's own launches.
//
// The launch sites wrap each kernel in ProfileScope; when profiling is enabled on this host
// thread the scope records a start/end CUDA event pair on the launch stream. Reading aggregates
// the pairs by kernel name. Only host-side event objects are created.
#include <algorithm>
#include <string>
#include <vector>

#include "kda_internal.h"

namespace kda {

struct ProfileRecord {
  const char* name;
  cudaEvent_t start, stop;
};

static thread_local bool t_prof_on = false;
static thread_local std::vector<ProfileRecord> t_prof_records;

ProfileScope::ProfileScope(const char* name, cudaStream_t stream) : name_(name), stream_(stream) {
  if (!t_prof_on) return;
  if (cudaEventCreate(&start_) != cudaSuccess) return;
  if (cudaEventCreate(&stop_) != cudaSuccess) {
    cudaEventDestroy(start_);
    return;
  }
  cudaEventRecord(start_, stream_);
  active_ = true;
}

ProfileScope::~ProfileScope() {
  if (!active_) return;
  cudaEventRecord(stop_, stream_);
  t_prof_records.push_back({name_, start_, stop_});
}

}  // namespace kda

extern "C" {

kda_status_t kda_profile_enable(int32_t enable) {
  kda::t_prof_on = enable != 0;
  return KDA_OK;
}

kda_status_t kda_profile_read(kda_profile_entry_t* entries, int32_t capacity, int32_t* count) {
  if (!count || capacity < 0 || (capacity > 0 && !entries)) return KDA_ERR_INVALID_ARG;
  struct Agg {
    std::string name;
    int32_t launches;
    double ms;
  };
  std::vector<Agg> agg;
  kda_status_t st = KDA_OK;
  for (auto& r : kda::t_prof_records) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess ||
        cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
      st = KDA_ERR_CUDA;
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
    auto it = std::find_if(agg.begin(), agg.end(), [&](const Agg& a) { return a.name == r.name; });
    if (it == agg.end()) {
      agg.push_back({r.name, 1, (double)ms});
    } else {
      it->launches += 1;
      it->ms += ms;
    }
  }
  kda::t_prof_records.clear();
  std::sort(agg.begin(), agg.end(), [](const Agg& a, const Agg& b) { return a.ms > b.ms; });
  *count = (int32_t)agg.size();
  for (int32_t i = 0; i < (int32_t)agg.size() && i < capacity; ++i) {
    snprintf(entries[i].name, sizeof(entries[i].name), "%s", agg[i].name.c_str());
    entries[i].launches = agg[i].launches;
    entries[i].total_ms = agg[i].ms;
  }
  return st;
}

}  // extern "C"
