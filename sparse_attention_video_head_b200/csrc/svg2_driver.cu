// Denoising-loop driver: the schedule the pages run around the layer (host code only).
//
// Over num_steps denoising steps and num_layers attention layers, the first dense_steps steps run
// dense attention (the pages keep full attention for the first denoising steps); at a layer's first
// sparse step its k-means starts cold (k-means++ and layer.iters Lloyd iterations); at its later
// steps it starts warm from the centroids that layer left at its previous sparse step (the pages'
// centroid cache across steps, "Key claims" section 4.3 and Fig. 7(a)), with warm_iters iterations.
// The driver owns host state only; the centroid cache is caller-owned device memory.
#include <new>
#include <vector>

#include "svg2.h"
#include "svg2_internal.h"

struct svg2_driver {
  svg2_driver_config cfg;
  int B, H, N, d;
  float* cache = nullptr;       // [num_layers][B*H*(nQ+nK)*d] float32, caller-owned device memory
  size_t cache_bytes = 0;
  std::vector<int> last_sparse; // per layer: the step of its last sparse call, -1 if its cache is cold
};

namespace {

size_t per_layer_floats(const svg2_driver* v) {
  return static_cast<size_t>(v->B) * v->H * (v->cfg.layer.nQ + v->cfg.layer.nK) * v->d;
}

int check_config(const svg2_driver_config* c, int B, int H, int N, int d) {
  if (c == nullptr) return SVG2_ERR_INVALID_ARG;
  if (c->num_steps < 1 || c->num_layers < 1 || c->dense_steps < 0 || c->dense_steps > c->num_steps)
    return SVG2_ERR_INVALID_ARG;
  if (c->warm_iters < 1 || c->layer.iters < 1) return SVG2_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return SVG2_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SVG2_ERR_UNSUPPORTED;
  if (c->layer.nQ < 1 || c->layer.nK < 1 || c->layer.nQ > N || c->layer.nK > N) return SVG2_ERR_INVALID_ARG;
  if (!(c->layer.top_p > 0.f) || !(c->layer.scale == c->layer.scale)) return SVG2_ERR_INVALID_ARG;
  return SVG2_OK;
}

}  // namespace

extern "C" {

int svg2_driver_create(const svg2_driver_config* cfg, int B, int H, int N, int d, svg2_driver** out) {
  if (out == nullptr) return SVG2_ERR_INVALID_ARG;
  *out = nullptr;
  const int r = check_config(cfg, B, H, N, d);
  if (r != SVG2_OK) return r;
  svg2_driver* v = new (std::nothrow) svg2_driver;
  if (v == nullptr) return SVG2_ERR_INVALID_ARG;
  try {
    v->cfg = *cfg;
    v->B = B;
    v->H = H;
    v->N = N;
    v->d = d;
    v->last_sparse.assign(static_cast<size_t>(cfg->num_layers), -1);
  } catch (...) {
    delete v;
    return SVG2_ERR_INVALID_ARG;
  }
  *out = v;
  return SVG2_OK;
}

int svg2_driver_destroy(svg2_driver* drv) {
  delete drv;
  return SVG2_OK;
}

int svg2_driver_cache_bytes(const svg2_driver* drv, size_t* bytes) {
  if (drv == nullptr || bytes == nullptr) return SVG2_ERR_INVALID_ARG;
  *bytes = per_layer_floats(drv) * sizeof(float) * static_cast<size_t>(drv->cfg.num_layers);
  return SVG2_OK;
}

int svg2_driver_bind_cache(svg2_driver* drv, float* cache, size_t bytes) {
  if (drv == nullptr || cache == nullptr) return SVG2_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(cache) % 16 != 0) return SVG2_ERR_INVALID_ARG;
  size_t need = 0;
  svg2_driver_cache_bytes(drv, &need);
  if (bytes < need) return SVG2_ERR_WORKSPACE;
  drv->cache = cache;
  drv->cache_bytes = bytes;
  for (auto& s : drv->last_sparse) s = -1;  // a new cache holds no centroids yet
  return SVG2_OK;
}

int svg2_driver_reset(svg2_driver* drv) {
  if (drv == nullptr) return SVG2_ERR_INVALID_ARG;
  for (auto& s : drv->last_sparse) s = -1;
  return SVG2_OK;
}

int svg2_driver_workspace_size(const svg2_driver* drv, size_t* bytes) {
  if (drv == nullptr || bytes == nullptr) return SVG2_ERR_INVALID_ARG;
  size_t a = 0, b = 0;
  int r = svg2_workspace_size(drv->B, drv->H, drv->N, drv->d, drv->cfg.layer.nQ, drv->cfg.layer.nK, &a);
  if (r != SVG2_OK) return r;
  if (drv->cfg.dense_steps > 0) {
    r = svg2_dense_attn_workspace_size(drv->B, drv->H, drv->N, drv->d, &b);
    if (r != SVG2_OK) return r;
  }
  *bytes = a > b ? a : b;
  return SVG2_OK;
}

int svg2_driver_plan(const svg2_driver* drv, int step, int layer, int* kind) {
  if (drv == nullptr || kind == nullptr) return SVG2_ERR_INVALID_ARG;
  if (step < 0 || step >= drv->cfg.num_steps || layer < 0 || layer >= drv->cfg.num_layers)
    return SVG2_ERR_INVALID_ARG;
  if (step < drv->cfg.dense_steps) *kind = SVG2_STEP_DENSE;
  else *kind = drv->last_sparse[static_cast<size_t>(layer)] < 0 ? SVG2_STEP_COLD : SVG2_STEP_WARM;
  return SVG2_OK;
}

int svg2_driver_layer(svg2_driver* drv, int step, int layer, const void* Q, const void* K, const void* V,
                      const double* uq, const double* uk, void* O, void* ws, size_t ws_bytes, void* stream) {
  int kind = 0;
  int r = svg2_driver_plan(drv, step, layer, &kind);
  if (r != SVG2_OK) return r;
  if (kind == SVG2_STEP_DENSE)
    return svg2_dense_attn(Q, K, V, drv->B, drv->H, drv->N, drv->d, drv->cfg.layer.scale, O, ws, ws_bytes, stream);
  if (drv->cache == nullptr) return SVG2_ERR_WORKSPACE;
  svg2_params p = drv->cfg.layer;
  if (kind == SVG2_STEP_COLD) {
    p.init = SVG2_INIT_KMEANSPP;
    if (uq == nullptr || uk == nullptr) return SVG2_ERR_INVALID_ARG;
  } else {
    p.init = SVG2_INIT_GIVEN;
    p.iters = drv->cfg.warm_iters;
  }
  float* cq = drv->cache + per_layer_floats(drv) * static_cast<size_t>(layer);
  float* ck = cq + static_cast<size_t>(drv->B) * drv->H * p.nQ * drv->d;
  r = svg2_layer(Q, K, V, SVG2_BF16, drv->B, drv->H, drv->N, drv->d, &p, uq, uk, cq, ck, O, nullptr, ws, ws_bytes,
                 stream);
  if (r == SVG2_OK) drv->last_sparse[static_cast<size_t>(layer)] = step;
  return r;
}

}  // extern "C"
