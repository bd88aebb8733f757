// The decode-step engine behind the C ABI of include/ocrdec.h.
//
// Host side only orders launches; every step of the decode path runs in the
// kernels of gemv.cuh, attention.cuh, route.cuh and step_kernels.cuh.  One
// verifier pass per layer is: Q/K/V GEMV (+RoPE, KV append) -> attention with
// the output projection (+residual; in MoE layers also the router partials)
// -> [dense SwiGLU up/down | expert gate/up GEMV that first routes the pass in
// every CTA, over the touched experts -> expert down GEMV -> combine].  Then
// final norm + LM head + argmax with acceptance in its last CTA.
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <new>
#include <tuple>
#include <vector>

#include "attention.cuh"
#include "launch.cuh"
#include "step_globals.cuh"

using namespace ocrdec;

namespace {

constexpr int kPrefillChunk = kRmax;  // context rows per prefill pass

// One weight matrix (or array of E expert matrices) with its tensor map.
struct Mat {
  const bf16* p = nullptr;
  int N = 0, K = 0, E = 1;
  CUtensorMap map;       // GEMV tiles
  CUtensorMap map_attn;  // W_o only: the attention kernel's per-(head, row block) boxes
};

struct LayerW {
  const bf16 *attn_norm, *ffn_norm;
  Mat wqkv, wo;
  Mat w_gu, w_down;                                 // dense layers
  Mat router, exp_gu, exp_down, sh_gu, sh_down;     // MoE layers
  bool dense;
};

struct DraftW {
  const bf16 *norm_h, *norm_e, *attn_norm, *ffn_norm, *final_norm;
  Mat fc, wqkv, wo, w_gu, w_down;
};

bool make_mat(Mat& m, const void* p, int N, int K, int E) {
  m.p = static_cast<const bf16*>(p);
  m.N = N;
  m.K = K;
  m.E = E;
  return encode_weight_map(p, K, N, E, &m.map) == cudaSuccess;
}

void manifest(const ocrdec_config& c, std::vector<std::vector<int64_t>>& m) {
  const int64_t d = c.d_model, V = c.vocab, E = c.n_experts, S = c.n_shared;
  m.clear();
  m.push_back({V, d});
  for (int l = 0; l < c.n_layers; ++l) {
    m.push_back({d});
    m.push_back({3 * d, d});
    m.push_back({d, d});
    m.push_back({d});
    if (l < c.n_dense_first) {
      m.push_back({2 * (int64_t)c.dense_ffn, d});
      m.push_back({d, c.dense_ffn});
    } else {
      m.push_back({E, d});
      m.push_back({E, 2 * (int64_t)c.expert_ffn, d});
      m.push_back({E, d, c.expert_ffn});
      m.push_back({S, 2 * (int64_t)c.shared_ffn, d});
      m.push_back({S, d, c.shared_ffn});
    }
  }
  m.push_back({d});
  m.push_back({V, d});
  m.push_back({d});
  m.push_back({d});
  m.push_back({d, 2 * d});
  m.push_back({d});
  m.push_back({3 * d, d});
  m.push_back({d, d});
  m.push_back({d});
  m.push_back({2 * (int64_t)c.draft_ffn, d});
  m.push_back({d, c.draft_ffn});
  m.push_back({d});
}

bool config_ok(const ocrdec_config* c) {
  if (!c) return false;
  const int pos[] = {c->d_model, c->n_layers, c->n_heads, c->head_dim, c->n_experts, c->top_k, c->expert_ffn,
                     c->shared_ffn, c->draft_ffn, c->vocab, c->max_batch, c->kv_capacity};
  for (int v : pos)
    if (v <= 0) return false;
  if (c->n_heads * c->head_dim != c->d_model) return false;
  if (c->head_dim != 64 && c->head_dim != 128) return false;
  // GEMV reduction dims are whole 64-column chunks; vocab rows need only 16-byte rows
  if (c->d_model % kChunk || c->expert_ffn % kChunk || c->draft_ffn % kChunk || c->vocab % 8) return false;
  if (c->n_dense_first < 0 || c->n_dense_first > c->n_layers) return false;
  if (c->n_dense_first > 0 && (c->dense_ffn <= 0 || c->dense_ffn % kChunk)) return false;
  if (c->n_shared < 0 || c->shared_ffn != c->expert_ffn) return false;
  // MoE layers: the down projection's rows of one item are copied whole (<= 1024 columns)
  if (c->n_dense_first < c->n_layers && c->expert_ffn > 1024) return false;
  if (c->top_k > c->n_experts || c->top_k > kMaxTopK || c->n_experts > kMaxExperts || c->n_shared > kMaxShared)
    return false;
  if (c->max_k < 0 || c->max_k > 3) return false;
  if (c->max_batch > kRmax || c->max_batch * (c->max_k + 1) > kRmax) return false;
  if (c->d_model > kGemvMaxK) return false;  // shared-memory copy of the normalised rows
  if (c->d_model > kAttnMaxD) return false;  // the attention block's W_qkv rows stay in shared memory
  // attention's fused output projection: d / 8 rows of W_o per CTA, whole 16-row MMA tiles, one TMA box
  if (c->d_model % (16 * kAttnSplit) || c->d_model / kAttnSplit > 256 || c->n_heads > kAttnMaxHeads) return false;
  if (c->kv_capacity > 8192) return false;  // documented limit of the C ABI
  if (!(c->rms_eps > 0.f) || !(c->rope_theta > 1.f)) return false;
  return true;
}

size_t align_up(size_t v) { return (v + 255) & ~(size_t)255; }

struct Layout {
  size_t status, counters, moe_ctr, tile_ctr, slots, rows, hist, rope, split_part, kvk, kvv, dkvk, dkvv, x, xd, q, yp,
      rpart, hbuf, hbuf_lo, ybuf, hdense, hdense_lo, fcin, fcin_lo,
      am_part, gtok, props,
      committed, ncommitted, hpend, total;
  int hist_ld, am_blocks;
};

Layout make_layout(const ocrdec_config& c, int am_blocks) {
  Layout L{};
  const size_t R = kRmax, B = c.max_batch, cap = c.kv_capacity, d = c.d_model, H = c.n_heads, Dh = c.head_dim;
  const size_t K = c.top_k, S = c.n_shared, f = c.expert_ffn;
  const size_t F = std::max(c.dense_ffn, c.draft_ffn);
  const size_t nslot = K + S;
  L.hist_ld = c.kv_capacity + 8;
  L.am_blocks = am_blocks;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
  L.status = take(256 + sizeof(TraceRec) * kTraceCap);  // status word + timeline trace
  L.counters = take(sizeof(int) * (16 + 2 * kWorkSlots + kRmax * kAttnSplit));
  L.moe_ctr = take(sizeof(int) * kMoeCtrInts);
  L.tile_ctr = take(sizeof(int) * kSplitMaxTiles);
  L.slots = take(sizeof(SlotState) * B);
  L.rows = take(sizeof(PassRows));
  L.hist = take(sizeof(int) * B * L.hist_ld);
  L.rope = take(sizeof(float2) * cap * (Dh / 2));
  L.split_part = take(sizeof(float) * kSplitPartFloats);
  L.kvk = take(2 * B * c.n_layers * H * cap * Dh);
  L.kvv = take(2 * B * c.n_layers * H * cap * Dh);
  L.dkvk = take(2 * B * H * cap * Dh);
  L.dkvv = take(2 * B * H * cap * Dh);
  L.x = take(4 * R * d);
  L.xd = take(4 * R * d);
  L.q = take(4 * R * d);
  L.yp = take(4 * H * kRmax * d);  // per-head output projections
  L.rpart = take(4 * R * kRouteParts * kRouteLd);
  L.hbuf = take(2 * R * nslot * f);
  L.hbuf_lo = take(2 * R * nslot * f);
  L.ybuf = take(4 * R * nslot * d);
  L.hdense = take(2 * R * F);
  L.hdense_lo = take(2 * R * F);
  L.fcin = take(2 * R * 2 * d);
  L.fcin_lo = take(2 * R * 2 * d);
  L.am_part = take(sizeof(float2) * am_blocks * kRmax);
  L.gtok = take(4 * R);
  L.props = take(4 * B * 4);
  L.committed = take(4 * B * 4);
  L.ncommitted = take(4 * B);
  L.hpend = take(4 * B * (c.max_k + 1) * d);
  L.total = o;
  return L;
}

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

template <class K>
cudaError_t max_carveout(K kernel) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
}

cudaError_t prepare_kernels_now() {
  cudaError_t e = cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)attn_smem_bytes(kAttnMaxD, kAttnMaxDh, kMaxExperts));
  // one shared-memory carveout for every kernel (no SM reconfiguration between launches)
  if (e == cudaSuccess) e = max_carveout(attention_kernel);
  if (e == cudaSuccess) e = max_carveout(verify_setup_kernel);
  if (e == cudaSuccess) e = max_carveout(prefill_setup_kernel);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(draft_setup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)draft_setup_smem_bytes(kGemvMaxK));
  if (e == cudaSuccess) e = max_carveout(draft_setup_kernel);
  if (e == cudaSuccess) e = max_carveout(accept_kernel);
  if (e == cudaSuccess) e = max_carveout(force_kernel);
  if (e == cudaSuccess) e = max_carveout(prefill_finish_kernel);
  if (e != cudaSuccess) return e;
  e = moe_prepare();
  if (e != cudaSuccess) return e;
  return gemv_prepare();
}

// Kernel attributes are per device: set them once for each device a call runs on.
cudaError_t prepare_kernels() {
  static std::mutex mu;
  static std::set<int> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count(dev)) return cudaSuccess;
  e = prepare_kernels_now();
  if (e == cudaSuccess) done.insert(dev);
  return e;
}

}  // namespace

struct ocrdec_ctx {
  ocrdec_config cfg;
  Layout L{};
  char* ws = nullptr;
  bool have_weights = false;
  int num_sms = 0;
  bool pdl = true;
  const bf16 *embed = nullptr, *final_norm = nullptr;
  Mat lm_head;
  std::vector<LayerW> layers;
  DraftW dw{};
  cudaStream_t cap_stream = nullptr;
  std::map<std::tuple<int, int, void*, void*>, cudaGraphExec_t> graphs;
  std::map<std::tuple<int, int, void*, void*>, int> graph_kernels;
  const int* f_ref = nullptr;
  const float* f_u = nullptr;
  const int* f_alt = nullptr;
  int f_npos = 0;
  float f_p[3] = {0, 0, 0};
  float* dbg_hidden = nullptr;
  float* dbg_logits = nullptr;
  float* dbg_draft_logits = nullptr;
  CUtensorMap kv_map[4];  // verifier K, V; draft K, V (encoded when the workspace is bound)
  // the draft's e4m3 copy of the LM head (variant; nullptr: the bf16 head)
  const unsigned char* head8 = nullptr;
  const float* head8_inv = nullptr;  // [V] inverse row scales
  CUtensorMap head8_map;

  template <class T>
  T* at(size_t off) const { return reinterpret_cast<T*>(ws + off); }
  int* status() const { return at<int>(L.status); }
  int* am_counter(int which) const { return at<int>(L.counters) + which; }
  // misc[0] = routed experts touched by verifier MoE layers, misc[1] = such layer passes
  int* misc() const { return at<int>(L.counters) + 8; }
  // attention / output-projection arrivals per (slot, row block)
  int* attn_counters() const { return at<int>(L.counters) + 16 + 2 * kWorkSlots; }
  // GEMV work counters, handed out round-robin so that launches next to each
  // other in a stream (which may overlap under programmatic dependent launch)
  // never share one; each launch's last CTA zeroes its pair
  mutable int work_next = 0;
  int* next_work() const {
    int* w = at<int>(L.counters) + 16 + 2 * work_next;
    work_next = (work_next + 1) % kWorkSlots;
    return w;
  }
  cudaError_t gemv(GemvLaunch& g, const LaunchCfg& lc) const {
    g.s.work = next_work();
    return launch_gemv(g, lc);
  }
  SlotState* slots() const { return at<SlotState>(L.slots); }
  PassRows* rows() const { return at<PassRows>(L.rows); }
  int* hist() const { return at<int>(L.hist); }
  LaunchCfg lc(cudaStream_t s) const { return LaunchCfg{s, pdl, num_sms}; }

  void drop_graphs() {
    for (auto& kv : graphs) cudaGraphExecDestroy(kv.second);
    graphs.clear();
    graph_kernels.clear();
  }
};

namespace {

#define CK(expr)                                   \
  do {                                             \
    cudaError_t e_ = (expr);                       \
    if (e_ != cudaSuccess) return OCRDEC_ECUDA;    \
  } while (0)

// ---------------------------------------------------------------------------
// building blocks
// ---------------------------------------------------------------------------

// Timeline-trace tags of the launches (ocrdec_read_trace).
enum Tag {
  kTagQKV = 1, kTagExpGU = 4, kTagExpDown = 5, kTagDenseGU = 6, kTagDenseDown = 7,
  kTagLMVerify = 8, kTagLMDraft = 9, kTagFC = 10
};

struct BlockIO {
  float* x;            // residual rows of the pass
  bf16* kc;            // K cache of this block, slot 0 (layer offset applied)
  bf16* vc;
  long long slot_stride;
  const CUtensorMap* tk;  // tensor maps over the whole K / V cache
  const CUtensorMap* tv;
  int layer, n_layers;    // this block's layer in the cache
};

// A GEMV launch over one dense matrix.
GemvLaunch dense_launch(ocrdec_ctx* c, const Mat& m, int pair_half, const int* nrows, int rows_static, int rmax,
                        int tag) {
  GemvLaunch g;
  g.s.tag = tag;
  g.tm_w = m.map;
  g.s.N = m.N;
  g.s.K = m.K;
  g.s.pair_half = pair_half;
  g.s.nrows = nrows;
  g.s.rows_static = rows_static;
  g.s.status = c->status();
  g.rows_bound = rmax;
  gemv_plan(g.s);
  g.s.kparts = gemv_kparts(g.s, 2 * c->num_sms);
  g.s.part = c->at<float>(c->L.split_part);
  g.s.tile_counter = c->at<int>(c->L.tile_ctr);
  return g;
}

// The attention block: RMSNorm, QKV + RoPE + KV append, attention, output
// projection and residual add in one clustered launch.  router / ffn_norm: a
// MoE layer's router and FFN norm gains (the kernel then also writes the router
// partials), or nullptr.  rows_pre_wait: the pass rows were written two or
// more kernels back, so the kernel may read them before its dependency wait.
int qkv_attn_oproj(ocrdec_ctx* c, const LaunchCfg& lc, const bf16* attn_norm, const Mat& wqkv, const Mat& wo,
                   const BlockIO& io, bool rows_pre_wait, const bf16* router = nullptr,
                   const bf16* ffn_norm = nullptr) {
  const ocrdec_config& m = c->cfg;
  PassRows* rows = c->rows();
  AttnParams a{};
  a.layer = io.layer;
  a.n_layers = io.n_layers;
  a.cap = m.kv_capacity;
  a.H = m.n_heads;
  a.Dh = m.head_dim;
  a.scale = 1.0f / std::sqrt((float)m.head_dim);
  a.slot_row0 = rows->slot_row0;
  a.slot_nrows = rows->slot_nrows;
  a.row_pos = rows->pos;
  a.rows_pre_wait = rows_pre_wait ? 1 : 0;
  a.x = io.x;
  a.yp = c->at<float>(c->L.yp);
  a.cnt = c->attn_counters();
  a.d = m.d_model;
  a.wqkv = wqkv.p;
  a.g_attn = attn_norm;
  a.eps = m.rms_eps;
  a.rope = c->at<float2>(c->L.rope);
  a.kc = io.kc;
  a.vc = io.vc;
  a.slot_stride = io.slot_stride;
  a.wr = router;
  a.g_ffn = ffn_norm;
  a.rpart = c->at<float>(c->L.rpart);
  a.E = m.n_experts;
  a.status = c->status();
  CK(launch_cluster_ex(attention_kernel, dim3(kAttnSplit, m.n_heads, m.max_batch), dim3(kAttnThreads),
                       attn_smem_bytes(m.d_model, m.head_dim, router ? m.n_experts : 0), lc, kAttnSplit, *io.tk,
                       *io.tv, wo.map_attn, a));
  return OCRDEC_OK;
}

int dense_ffn(ocrdec_ctx* c, const LaunchCfg& lc, int rmax, float* x, const bf16* norm, const Mat& w_gu,
              const Mat& w_down) {
  const ocrdec_config& m = c->cfg;
  PassRows* rows = c->rows();
  const int F = w_down.K;
  bf16* h = c->at<bf16>(c->L.hdense);
  GemvLaunch g = dense_launch(c, w_gu, F, &rows->n, 0, rmax, kTagDenseGU);
  g.src = SrcKind::Norm;
  g.norm = SrcNorm::Params{x, m.d_model, nullptr, norm, m.rms_eps};
  g.epi = EpiKind::SwiGLU;
  g.swiglu = EpiSwiGLU::Params{h, c->at<bf16>(c->L.hdense_lo), F, 1};
  CK(c->gemv(g, lc));

  GemvLaunch dn = dense_launch(c, w_down, 0, &rows->n, 0, rmax, kTagDenseDown);
  dn.src = SrcKind::Bf16;
  dn.bf = SrcBf16::Params{h, c->at<bf16>(c->L.hdense_lo), F, 1, nullptr};
  dn.epi = EpiKind::StoreAdd;
  dn.store = EpiStore<false>::Params{x, m.d_model, 1, nullptr};
  CK(c->gemv(dn, lc));
  return OCRDEC_OK;
}

int moe_ffn(ocrdec_ctx* c, const LaunchCfg& lc, int rmax, const LayerW& w, bool count) {
  const ocrdec_config& m = c->cfg;
  // routing, shared + routed experts and the combine: one persistent kernel
  MoeLaunch g;
  g.tm_gu = w.exp_gu.map;
  g.tm_sgu = w.sh_gu.map;
  g.tm_dn = w.exp_down.map;
  g.tm_sdn = w.sh_down.map;
  MoeParams& p = g.p;
  p.d = m.d_model;
  p.f = m.expert_ffn;
  p.E = m.n_experts;
  p.S = m.n_shared;
  p.top_k = m.top_k;
  p.tiles_gu = m.expert_ffn / kBoxRows;
  p.tiles_dn = m.d_model / kTile;
  p.eps = m.rms_eps;
  p.x = c->at<float>(c->L.x);
  p.nrows = &c->rows()->n;
  p.gain = w.ffn_norm;
  p.rpart = c->at<float>(c->L.rpart);
  p.h = c->at<bf16>(c->L.hbuf);
  p.h_lo = c->at<bf16>(c->L.hbuf_lo);
  p.y = c->at<float>(c->L.ybuf);
  p.ctr = c->at<int>(c->L.moe_ctr);
  p.touched = count ? c->misc() : nullptr;
  p.status = c->status();
  CK(launch_moe(g, rmax, lc));
  return OCRDEC_OK;
}

// All verifier layers over the rows prepared in x / rows.
int verifier_layers(ocrdec_ctx* c, const LaunchCfg& lc, int rmax, bool count) {
  const ocrdec_config& m = c->cfg;
  const long long layer_elems = (long long)m.n_heads * m.kv_capacity * m.head_dim;
  for (int l = 0; l < m.n_layers; ++l) {
    const LayerW& w = c->layers[l];
    BlockIO io{c->at<float>(c->L.x), c->at<bf16>(c->L.kvk) + l * layer_elems, c->at<bf16>(c->L.kvv) + l * layer_elems,
               layer_elems * m.n_layers, &c->kv_map[0], &c->kv_map[1], l, m.n_layers};
    // layer 0 follows the pass's setup kernel: its rows are read after the wait
    int st = qkv_attn_oproj(c, lc, w.attn_norm, w.wqkv, w.wo, io, l > 0, w.dense ? nullptr : w.router.p,
                            w.ffn_norm);
    if (st) return st;
    st = w.dense ? dense_ffn(c, lc, rmax, io.x, w.ffn_norm, w.w_gu, w.w_down) : moe_ffn(c, lc, rmax, w, count);
    if (st) return st;
    if (c->dbg_hidden)
      CK(cudaMemcpyAsync(c->dbg_hidden + (size_t)l * kRmax * m.d_model, io.x, sizeof(float) * kRmax * m.d_model,
                         cudaMemcpyDeviceToDevice, lc.stream));
  }
  return OCRDEC_OK;
}

// final norm + LM head + argmax.  row_src selects x rows (nullptr: rows 0..);
// nrows / rows_static the row count; tokens to tok[r * tok_stride].
int lm_head(ocrdec_ctx* c, const LaunchCfg& lc, int rmax, const float* x, const bf16* norm, const int* row_src,
            const int* nrows, int rows_static, int* tok, int tok_stride, float* logits, int which_counter,
            bool fp8 = false) {
  const ocrdec_config& m = c->cfg;
  GemvLaunch g = dense_launch(c, c->lm_head, 0, nrows, rows_static, rmax, kTagLMDraft);
  g.s.counter = c->am_counter(which_counter);
  g.src = SrcKind::Norm;
  if (fp8) {
    // the e4m3 head: K counted in byte pairs, logits scaled back per row
    g.tm_w = c->head8_map;
    g.s.K = m.d_model / 2;
    gemv_plan(g.s);
    g.s.kparts = 1;
    g.src = SrcKind::Norm8;
  }
  g.norm = SrcNorm::Params{x, m.d_model, row_src, norm, m.rms_eps};
  g.epi = EpiKind::Argmax;
  g.argmax = EpiArgmax::Params{tok, tok_stride, logits, c->at<float2>(c->L.am_part), nullptr,
                               fp8 ? c->head8_inv : nullptr};
  g.grid = std::min(g.s.tiles_per_mat, c->L.am_blocks);
  CK(c->gemv(g, lc));
  return OCRDEC_OK;
}

// The draft block over the rows prepared by draft_setup (fcin, rows).
// kv_only: stop after the draft KV append (prefill pairs whose outputs are unused).
int draft_block(ocrdec_ctx* c, const LaunchCfg& lc, int rmax, bool kv_only, int* tok, int tok_stride, int j) {
  const ocrdec_config& m = c->cfg;
  const DraftW& w = c->dw;
  PassRows* rows = c->rows();
  float* xd = c->at<float>(c->L.xd);
  GemvLaunch fc = dense_launch(c, w.fc, 0, &rows->n, 0, rmax, kTagFC);
  fc.src = SrcKind::Bf16;
  fc.bf = SrcBf16::Params{c->at<bf16>(c->L.fcin), c->at<bf16>(c->L.fcin_lo), 2 * m.d_model, 1, nullptr};
  fc.epi = EpiKind::Store;
  fc.store = EpiStore<false>::Params{xd, m.d_model, 1, nullptr};
  CK(c->gemv(fc, lc));

  const long long slot_elems = (long long)m.n_heads * m.kv_capacity * m.head_dim;
  BlockIO io{xd, c->at<bf16>(c->L.dkvk), c->at<bf16>(c->L.dkvv), slot_elems, &c->kv_map[2], &c->kv_map[3], 0, 1};
  if (kv_only) {
    GemvLaunch g = dense_launch(c, w.wqkv, m.head_dim / 2, &rows->n, 0, rmax, kTagQKV);
    g.src = SrcKind::Norm;
    g.norm = SrcNorm::Params{xd, m.d_model, nullptr, w.attn_norm, m.rms_eps};
    g.epi = EpiKind::QKV;
    g.qkv = EpiQKV::Params{c->at<float>(c->L.q), io.kc, io.vc, io.slot_stride, m.kv_capacity, m.n_heads,
                           m.head_dim, c->at<float2>(c->L.rope), rows->slot, rows->pos};
    CK(c->gemv(g, lc));
    return OCRDEC_OK;
  }
  int st = qkv_attn_oproj(c, lc, w.attn_norm, w.wqkv, w.wo, io, true);  // draft setup, fc, then this
  if (st) return st;
  st = dense_ffn(c, lc, rmax, xd, w.ffn_norm, w.w_gu, w.w_down);
  if (st) return st;
  float* dl = c->dbg_draft_logits ? c->dbg_draft_logits + (size_t)(j - 1) * m.max_batch * m.vocab : nullptr;
  return lm_head(c, lc, m.max_batch, xd, w.final_norm, rows->last_row, &rows->n_last, 0, tok, tok_stride, dl, 1,
                 c->head8 != nullptr);
}

int enqueue_draft(ocrdec_ctx* c, const LaunchCfg& lc, int B, int k, int* props) {
  const ocrdec_config& m = c->cfg;
  for (int j = 1; j <= k; ++j) {
    DraftSetupParams dp{};
    dp.mode = j == 1 ? 0 : 1;
    dp.B = B;
    dp.j = j;
    dp.d = m.d_model;
    dp.max_k = m.max_k;
    dp.eps = m.rms_eps;
    dp.slots = c->slots();
    dp.hist = c->hist();
    dp.hist_ld = c->L.hist_ld;
    dp.hpend = c->at<float>(c->L.hpend);
    dp.xd = c->at<float>(c->L.xd);
    dp.dtok = props + (j >= 2 ? j - 2 : 0);
    dp.dtok_stride = k;
    dp.embed = c->embed;
    dp.g_h = c->dw.norm_h;
    dp.g_e = c->dw.norm_e;
    dp.fcin = c->at<bf16>(c->L.fcin);
    dp.fcin_lo = c->at<bf16>(c->L.fcin_lo);
    dp.rows = c->rows();
    dp.rows_prev = c->rows();
    dp.status = c->status();
    CK(launch_ex(draft_setup_kernel, dim3(1), dim3(256), draft_setup_smem_bytes(m.d_model), lc, dp));
    int rmax = j == 1 ? std::min(kRmax, B * (m.max_k + 1)) : B;
    int st = draft_block(c, lc, rmax, false, props + (j - 1), k, j);
    if (st) return st;
  }
  return OCRDEC_OK;
}

int enqueue_force(ocrdec_ctx* c, const LaunchCfg& lc, int B, int k, int* props) {
  if (!c->f_ref || k == 0) return OCRDEC_OK;
  ForceParams fp{c->slots(), props, B, k, c->cfg.max_k, c->f_ref, c->f_u, c->f_alt, c->f_npos,
                 c->f_p[0], c->f_p[1], c->f_p[2], c->status()};
  CK(launch_ex(force_kernel, dim3(1), dim3(32), 0, lc, fp));
  return OCRDEC_OK;
}

int enqueue_verify(ocrdec_ctx* c, const LaunchCfg& lc, int B, int k, const int* props, int* committed,
                   int* ncommitted) {
  const ocrdec_config& m = c->cfg;
  const int R = B * (k + 1);
  VerifySetupParams vp{c->slots(), props, B, k, m.kv_capacity, m.d_model, m.vocab, c->embed,
                       c->at<float>(c->L.x), c->rows(), c->status()};
  CK(launch_ex(verify_setup_kernel, dim3(1), dim3(256), 0, lc, vp));
  int st = verifier_layers(c, lc, R, true);
  if (st) return st;
  AcceptParams ap{c->slots(), c->at<int>(c->L.gtok), props, B, k, m.d_model, m.max_k, c->hist(), c->L.hist_ld,
                  c->at<float>(c->L.x), c->at<float>(c->L.hpend), committed, ncommitted, c->status()};
  GemvLaunch g = dense_launch(c, c->lm_head, 0, &c->rows()->n, 0, R, kTagLMVerify);
  g.s.counter = c->am_counter(0);
  g.src = SrcKind::Norm;
  g.norm = SrcNorm::Params{c->at<float>(c->L.x), m.d_model, nullptr, c->final_norm, m.rms_eps};
  g.epi = EpiKind::ArgmaxAccept;
  g.argmax = EpiArgmax::Params{c->at<int>(c->L.gtok), 1, c->dbg_logits, c->at<float2>(c->L.am_part), nullptr};
  g.accept = ap;
  g.grid = std::min(g.s.tiles_per_mat, c->L.am_blocks);
  CK(c->gemv(g, lc));
  return OCRDEC_OK;
}

int enqueue_step(ocrdec_ctx* c, const LaunchCfg& lc, int B, int k, int* committed, int* ncommitted) {
  int* props = c->at<int>(c->L.props);
  int st = OCRDEC_OK;
  if (k > 0) {
    st = enqueue_draft(c, lc, B, k, props);
    if (st) return st;
    st = enqueue_force(c, lc, B, k, props);
    if (st) return st;
  }
  return enqueue_verify(c, lc, B, k, props, committed, ncommitted);
}

// Scratch of the single-kernel entry points: status word, trace header (kept
// zero: tracing off), last-block counter at word 8, argmax partials, split-K
// tile counters and partial sums.  Returns the byte size.
size_t op_scratch_layout(int sms, size_t* am, size_t* ctr, size_t* part) {
  size_t o = 256;
  if (am) *am = o;
  o = align_up(o + sizeof(float2) * 2 * sms * kRmax);
  if (ctr) *ctr = o;
  o = align_up(o + sizeof(int) * kSplitMaxTiles);
  if (part) *part = o;
  return align_up(o + sizeof(float) * kSplitPartFloats);
}

int check_ready(const ocrdec_ctx* c) {
  if (!c) return OCRDEC_EINVAL;
  if (!c->ws || !c->have_weights) return OCRDEC_ESTATE;
  return OCRDEC_OK;
}

int check_bk(const ocrdec_ctx* c, int batch, int k) {
  if (batch < 1 || batch > c->cfg.max_batch || k < 0 || k > c->cfg.max_k) return OCRDEC_EINVAL;
  if (batch * (k + 1) > kRmax) return OCRDEC_EINVAL;
  return OCRDEC_OK;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

int ocrdec_create(const ocrdec_config* cfg, ocrdec_ctx** out) {
  if (!out) return OCRDEC_EINVAL;
  *out = nullptr;
  if (!config_ok(cfg)) return OCRDEC_EINVAL;
  ocrdec_ctx* c = new (std::nothrow) ocrdec_ctx();
  if (!c) return OCRDEC_ENOMEM;
  c->cfg = *cfg;
  c->num_sms = device_sms();
  if (c->num_sms <= 0) c->num_sms = 148;
  c->L = make_layout(*cfg, 2 * c->num_sms);
  *out = c;
  return OCRDEC_OK;
}

void ocrdec_destroy(ocrdec_ctx* c) {
  if (!c) return;
  c->drop_graphs();
  if (c->cap_stream) cudaStreamDestroy(c->cap_stream);
  delete c;
}

int ocrdec_weight_count(const ocrdec_config* cfg) {
  if (!config_ok(cfg)) return -OCRDEC_EINVAL;
  std::vector<std::vector<int64_t>> m;
  manifest(*cfg, m);
  return (int)m.size();
}

int ocrdec_weight_info(const ocrdec_config* cfg, int index, int64_t dims[3], int32_t* ndim) {
  if (!config_ok(cfg) || !dims || !ndim) return OCRDEC_EINVAL;
  std::vector<std::vector<int64_t>> m;
  manifest(*cfg, m);
  if (index < 0 || index >= (int)m.size()) return OCRDEC_EINVAL;
  *ndim = (int32_t)m[index].size();
  for (int i = 0; i < 3; ++i) dims[i] = i < *ndim ? m[index][i] : 0;
  return OCRDEC_OK;
}

size_t ocrdec_workspace_bytes(const ocrdec_config* cfg) {
  if (!config_ok(cfg)) return 0;
  int sms = device_sms();
  return make_layout(*cfg, 2 * (sms > 0 ? sms : 148)).total;
}

int ocrdec_bind_workspace(ocrdec_ctx* c, void* ws, size_t bytes, ocrdec_stream stream) {
  if (!c || !ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return OCRDEC_EINVAL;
  if (bytes < c->L.total) return OCRDEC_ENOMEM;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  c->ws = static_cast<char*>(ws);
  c->drop_graphs();
  CK(prepare_kernels());
  // status, counters, slots, rows and token history start at zero; so do the
  // KV caches, whose unwritten positions attention reads (with weight 0)
  CK(cudaMemsetAsync(c->ws, 0, c->L.rope, s));
  CK(cudaMemsetAsync(c->ws + c->L.kvk, 0, c->L.x - c->L.kvk, s));
  {
    const ocrdec_config& mc = c->cfg;
    const int B = mc.max_batch;
    const void* bases[4] = {c->ws + c->L.kvk, c->ws + c->L.kvv, c->ws + c->L.dkvk, c->ws + c->L.dkvv};
    for (int i = 0; i < 4; ++i)
      CK(encode_kv_map(bases[i], mc.head_dim, mc.kv_capacity, mc.n_heads, i < 2 ? B * mc.n_layers : B, &c->kv_map[i]));
  }
  const ocrdec_config& m = c->cfg;
  long long n = (long long)m.kv_capacity * (m.head_dim / 2);
  rope_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(c->at<float2>(c->L.rope), m.kv_capacity, m.head_dim,
                                                                  (double)m.rope_theta);
  CK(cudaGetLastError());
  if (!c->cap_stream) CK(cudaStreamCreateWithFlags(&c->cap_stream, cudaStreamNonBlocking));
  return OCRDEC_OK;
}

int ocrdec_load_weights(ocrdec_ctx* c, const void* const* ptrs, int n) {
  if (!c || !ptrs) return OCRDEC_EINVAL;
  const ocrdec_config& m = c->cfg;
  std::vector<std::vector<int64_t>> man;
  manifest(m, man);
  if (n != (int)man.size()) return OCRDEC_EINVAL;
  for (int i = 0; i < n; ++i)
    if (!ptrs[i] || (reinterpret_cast<uintptr_t>(ptrs[i]) & 15)) return OCRDEC_EINVAL;
  auto W = [&](int i) { return static_cast<const bf16*>(ptrs[i]); };
  const int d = m.d_model;
  bool ok = true;
  int i = 0;
  c->embed = W(i++);
  c->layers.assign(m.n_layers, LayerW{});
  for (int l = 0; l < m.n_layers; ++l) {
    LayerW& L = c->layers[l];
    L.attn_norm = W(i++);
    ok &= make_mat(L.wqkv, W(i++), 3 * d, d, 1);
    ok &= make_mat(L.wo, W(i++), d, d, 1);
    ok &= encode_oproj_map(L.wo.p, d, m.head_dim, &L.wo.map_attn) == cudaSuccess;
    L.ffn_norm = W(i++);
    L.dense = l < m.n_dense_first;
    if (L.dense) {
      ok &= make_mat(L.w_gu, W(i++), 2 * m.dense_ffn, d, 1);
      ok &= make_mat(L.w_down, W(i++), d, m.dense_ffn, 1);
    } else {
      ok &= make_mat(L.router, W(i++), m.n_experts, d, 1);
      ok &= make_mat(L.exp_gu, W(i++), 2 * m.expert_ffn, d, m.n_experts);
      ok &= make_mat(L.exp_down, W(i++), d, m.expert_ffn, m.n_experts);
      if (m.n_shared > 0) {
        ok &= make_mat(L.sh_gu, W(i++), 2 * m.shared_ffn, d, m.n_shared);
        ok &= make_mat(L.sh_down, W(i++), d, m.shared_ffn, m.n_shared);
      } else {
        i += 2;
        L.sh_gu = L.exp_gu;
        L.sh_down = L.exp_down;
      }
    }
  }
  c->final_norm = W(i++);
  ok &= make_mat(c->lm_head, W(i++), m.vocab, d, 1);
  DraftW& dw = c->dw;
  dw.norm_h = W(i++);
  dw.norm_e = W(i++);
  ok &= make_mat(dw.fc, W(i++), d, 2 * d, 1);
  dw.attn_norm = W(i++);
  ok &= make_mat(dw.wqkv, W(i++), 3 * d, d, 1);
  ok &= make_mat(dw.wo, W(i++), d, d, 1);
  ok &= encode_oproj_map(dw.wo.p, d, m.head_dim, &dw.wo.map_attn) == cudaSuccess;
  dw.ffn_norm = W(i++);
  ok &= make_mat(dw.w_gu, W(i++), 2 * m.draft_ffn, d, 1);
  ok &= make_mat(dw.w_down, W(i++), d, m.draft_ffn, 1);
  dw.final_norm = W(i++);
  if (!ok) return OCRDEC_ECUDA;
  c->have_weights = true;
  c->drop_graphs();
  return OCRDEC_OK;
}

int ocrdec_prefill(ocrdec_ctx* c, int slot, const float* visual, int n_visual, const int32_t* prompt, int n_prompt,
                   int32_t* first_token, ocrdec_stream stream) {
  int st = check_ready(c);
  if (st) return st;
  const ocrdec_config& m = c->cfg;
  const int C = n_visual + n_prompt;
  if (slot < 0 || slot >= m.max_batch || n_visual < 0 || n_prompt < 0 || C < 1) return OCRDEC_EINVAL;
  if ((n_visual > 0 && !visual) || (n_prompt > 0 && !prompt)) return OCRDEC_EINVAL;
  if (C + m.max_k + 2 > m.kv_capacity) return OCRDEC_ECAPACITY;
  LaunchCfg lc = c->lc(reinterpret_cast<cudaStream_t>(stream));
  for (int p0 = 0; p0 < C; p0 += kPrefillChunk) {
    const int n = std::min(kPrefillChunk, C - p0);
    PrefillSetupParams ps{slot, p0, n, n_visual, m.vocab, n_prompt, visual, prompt, c->embed, m.d_model,
                          c->at<float>(c->L.x), c->rows(), c->status()};
    CK(launch_ex(prefill_setup_kernel, dim3(1), dim3(256), 0, lc, ps));
    st = verifier_layers(c, lc, n, false);
    if (st) return st;
    if (p0 + n == C) {
      st = lm_head(c, lc, 1, c->at<float>(c->L.x), c->final_norm, c->rows()->last_row, nullptr, 1,
                   c->at<int>(c->L.gtok), 1, nullptr, 0);
      if (st) return st;
    }
    const int q1 = std::min(p0 + n, C - 1);
    if (q1 > p0) {
      DraftSetupParams dp{};
      dp.mode = 2;
      dp.B = 1;
      dp.d = m.d_model;
      dp.max_k = m.max_k;
      dp.eps = m.rms_eps;
      dp.slots = c->slots();
      dp.slot = slot;
      dp.p0 = p0;
      dp.n = q1 - p0;
      dp.n_visual = n_visual;
      dp.xv = c->at<float>(c->L.x);
      dp.visual = visual;
      dp.prompt = prompt;
      dp.embed = c->embed;
      dp.g_h = c->dw.norm_h;
      dp.g_e = c->dw.norm_e;
      dp.fcin = c->at<bf16>(c->L.fcin);
      dp.fcin_lo = c->at<bf16>(c->L.fcin_lo);
    dp.fcin_lo = c->at<bf16>(c->L.fcin_lo);
      dp.rows = c->rows();
      dp.rows_prev = c->rows();
      dp.status = c->status();
      // the verifier rows of this chunk are needed by the draft setup and, on the
      // last chunk, by the finish step: run the finish first when both apply
      if (p0 + n == C) {
        PrefillFinishParams pf{c->slots(), slot, C, C - 1 - p0, m.d_model, m.max_k, c->at<int>(c->L.gtok),
                               c->at<float>(c->L.x), c->at<float>(c->L.hpend), c->hist(), c->L.hist_ld,
                               first_token, c->status()};
        CK(launch_ex(prefill_finish_kernel, dim3(1), dim3(256), 0, lc, pf));
      }
      CK(launch_ex(draft_setup_kernel, dim3(1), dim3(256), draft_setup_smem_bytes(m.d_model), lc, dp));
      st = draft_block(c, lc, q1 - p0, true, nullptr, 0, 0);
      if (st) return st;
    } else if (p0 + n == C) {
      PrefillFinishParams pf{c->slots(), slot, C, C - 1 - p0, m.d_model, m.max_k, c->at<int>(c->L.gtok),
                             c->at<float>(c->L.x), c->at<float>(c->L.hpend), c->hist(), c->L.hist_ld,
                             first_token, c->status()};
      CK(launch_ex(prefill_finish_kernel, dim3(1), dim3(256), 0, lc, pf));
    }
  }
  return OCRDEC_OK;
}

int ocrdec_draft(ocrdec_ctx* c, int batch, int k, int32_t* props, ocrdec_stream stream) {
  int st = check_ready(c);
  if (st) return st;
  if ((st = check_bk(c, batch, k))) return st;
  if (k < 1 || !props) return OCRDEC_EINVAL;
  return enqueue_draft(c, c->lc(reinterpret_cast<cudaStream_t>(stream)), batch, k, props);
}

int ocrdec_verify_commit(ocrdec_ctx* c, int batch, int k, const int32_t* props, int32_t* committed,
                         int32_t* ncommitted, ocrdec_stream stream) {
  int st = check_ready(c);
  if (st) return st;
  if ((st = check_bk(c, batch, k))) return st;
  if ((k > 0 && !props) || !committed || !ncommitted) return OCRDEC_EINVAL;
  return enqueue_verify(c, c->lc(reinterpret_cast<cudaStream_t>(stream)), batch, k, props, committed, ncommitted);
}

int ocrdec_step(ocrdec_ctx* c, int batch, int k, int32_t* committed, int32_t* ncommitted, ocrdec_stream stream) {
  int st = check_ready(c);
  if (st) return st;
  if ((st = check_bk(c, batch, k))) return st;
  if (!committed || !ncommitted) return OCRDEC_EINVAL;
  auto key = std::make_tuple(batch, k, (void*)committed, (void*)ncommitted);
  auto itg = c->graphs.find(key);
  cudaGraphExec_t exec = nullptr;
  if (itg == c->graphs.end()) {
    cudaGraph_t graph = nullptr;
    CK(cudaStreamBeginCapture(c->cap_stream, cudaStreamCaptureModeThreadLocal));
    st = enqueue_step(c, c->lc(c->cap_stream), batch, k, committed, ncommitted);
    cudaError_t e = cudaStreamEndCapture(c->cap_stream, &graph);
    if (st) {
      if (graph) cudaGraphDestroy(graph);
      return st;
    }
    if (e != cudaSuccess) return OCRDEC_ECUDA;
    size_t nn = 0;
    int nk = 0;
    if (cudaGraphGetNodes(graph, nullptr, &nn) == cudaSuccess && nn > 0) {
      std::vector<cudaGraphNode_t> nodes(nn);
      if (cudaGraphGetNodes(graph, nodes.data(), &nn) == cudaSuccess)
        for (auto nd : nodes) {
          cudaGraphNodeType t;
          if (cudaGraphNodeGetType(nd, &t) == cudaSuccess && t == cudaGraphNodeTypeKernel) ++nk;
        }
    }
    c->graph_kernels[key] = nk;
    e = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) return OCRDEC_ECUDA;
    c->graphs[key] = exec;
  } else {
    exec = itg->second;
  }
  CK(cudaGraphLaunch(exec, reinterpret_cast<cudaStream_t>(stream)));
  return OCRDEC_OK;
}

int ocrdec_step_host(ocrdec_ctx* c, int batch, int k, int32_t* host_committed, int32_t* host_n, ocrdec_stream stream) {
  int st = check_ready(c);
  if (st) return st;
  if (!host_committed || !host_n) return OCRDEC_EINVAL;
  int* dc = c->at<int>(c->L.committed);
  int* dn = c->at<int>(c->L.ncommitted);
  if ((st = ocrdec_step(c, batch, k, dc, dn, stream))) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  CK(cudaMemcpyAsync(host_committed, dc, sizeof(int) * batch * (k + 1), cudaMemcpyDeviceToHost, s));
  CK(cudaMemcpyAsync(host_n, dn, sizeof(int) * batch, cudaMemcpyDeviceToHost, s));
  CK(cudaStreamSynchronize(s));
  return OCRDEC_OK;
}

int ocrdec_set_forced_acceptance(ocrdec_ctx* c, const int32_t* ref, const float* u, const int32_t* alt, int n_pos,
                                 const float* host_p) {
  if (!c) return OCRDEC_EINVAL;
  c->drop_graphs();
  if (!ref) {
    c->f_ref = nullptr;
    return OCRDEC_OK;
  }
  if (!u || !alt || n_pos <= 0 || !host_p) return OCRDEC_EINVAL;
  c->f_ref = ref;
  c->f_u = u;
  c->f_alt = alt;
  c->f_npos = n_pos;
  for (int j = 0; j < 3; ++j) c->f_p[j] = j < c->cfg.max_k ? host_p[j] : 0.f;
  return OCRDEC_OK;
}

int ocrdec_get_status(ocrdec_ctx* c, int32_t* host_status, ocrdec_stream stream) {
  if (!c || !host_status) return OCRDEC_EINVAL;
  if (!c->ws) return OCRDEC_ESTATE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  CK(cudaMemcpyAsync(host_status, c->status(), sizeof(int), cudaMemcpyDeviceToHost, s));
  CK(cudaStreamSynchronize(s));
  return OCRDEC_OK;
}

int ocrdec_clear_status(ocrdec_ctx* c, ocrdec_stream stream) {
  if (!c) return OCRDEC_EINVAL;
  if (!c->ws) return OCRDEC_ESTATE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  CK(cudaMemsetAsync(c->status(), 0, sizeof(int), s));
  // arrival counters that an aborted launch may have left part-way
  CK(cudaMemsetAsync(c->am_counter(0), 0, 8 * sizeof(int), s));
  CK(cudaMemsetAsync(c->at<int>(c->L.counters) + 16, 0, (2 * kWorkSlots + kRmax * kAttnSplit) * sizeof(int), s));
  CK(cudaMemsetAsync(c->at<int>(c->L.tile_ctr), 0, kSplitMaxTiles * sizeof(int), s));
  CK(cudaMemsetAsync(c->at<int>(c->L.moe_ctr), 0, kMoeCtrInts * sizeof(int), s));
  return OCRDEC_OK;
}

int ocrdec_get_slot_stats(ocrdec_ctx* c, int slot, ocrdec_slot_stats* out, ocrdec_stream stream) {
  if (!c || !out || slot < 0 || slot >= c->cfg.max_batch) return OCRDEC_EINVAL;
  if (!c->ws) return OCRDEC_ESTATE;
  static_assert(sizeof(ocrdec_slot_stats) == 10 * sizeof(int32_t), "stats layout");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  CK(cudaMemcpyAsync(out, c->slots() + slot, sizeof(ocrdec_slot_stats), cudaMemcpyDeviceToHost, s));
  CK(cudaStreamSynchronize(s));
  return OCRDEC_OK;
}

int ocrdec_token_history(ocrdec_ctx* c, int slot, const int32_t** dev_tokens) {
  if (!c || !dev_tokens || slot < 0 || slot >= c->cfg.max_batch) return OCRDEC_EINVAL;
  if (!c->ws) return OCRDEC_ESTATE;
  *dev_tokens = c->hist() + (size_t)slot * c->L.hist_ld;
  return OCRDEC_OK;
}

int ocrdec_get_counters(ocrdec_ctx* c, int32_t* host, int n, ocrdec_stream stream) {
  if (!c || !host || n < 1 || n > 2) return OCRDEC_EINVAL;
  if (!c->ws) return OCRDEC_ESTATE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  CK(cudaMemcpyAsync(host, c->misc(), sizeof(int32_t) * n, cudaMemcpyDeviceToHost, s));
  CK(cudaStreamSynchronize(s));
  return OCRDEC_OK;
}

int ocrdec_reset_counters(ocrdec_ctx* c, ocrdec_stream stream) {
  if (!c) return OCRDEC_EINVAL;
  if (!c->ws) return OCRDEC_ESTATE;
  CK(cudaMemsetAsync(c->misc(), 0, 2 * sizeof(int32_t), reinterpret_cast<cudaStream_t>(stream)));
  return OCRDEC_OK;
}

int ocrdec_step_kernel_count(ocrdec_ctx* c, int batch, int k, int32_t* dev_committed, int32_t* dev_n_committed,
                             int32_t* count) {
  if (!c || !count) return OCRDEC_EINVAL;
  auto it = c->graph_kernels.find(std::make_tuple(batch, k, (void*)dev_committed, (void*)dev_n_committed));
  if (it == c->graph_kernels.end()) return OCRDEC_ESTATE;
  *count = it->second;
  return OCRDEC_OK;
}

int ocrdec_set_trace(ocrdec_ctx* c, int enable, ocrdec_stream stream) {
  if (!c) return OCRDEC_EINVAL;
  if (!c->ws) return OCRDEC_ESTATE;
  int v[2] = {enable ? 1 : 0, 0};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  CK(cudaMemcpyAsync(c->status() + 1, v, sizeof(v), cudaMemcpyHostToDevice, s));
  CK(cudaStreamSynchronize(s));
  return OCRDEC_OK;
}

int ocrdec_read_trace(ocrdec_ctx* c, void* host_records, int max_records, int32_t* n, ocrdec_stream stream) {
  if (!c || !n || max_records < 0 || (max_records > 0 && !host_records)) return OCRDEC_EINVAL;
  if (!c->ws) return OCRDEC_ESTATE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int cnt = 0;
  CK(cudaMemcpyAsync(&cnt, c->status() + 2, sizeof(cnt), cudaMemcpyDeviceToHost, s));
  CK(cudaStreamSynchronize(s));
  int take = (int)std::min<unsigned>(std::min<unsigned>(cnt, (unsigned)kTraceCap), (unsigned)max_records);
  if (take > 0)
    CK(cudaMemcpyAsync(host_records, reinterpret_cast<char*>(c->status()) + 256, sizeof(TraceRec) * take,
                       cudaMemcpyDeviceToHost, s));
  CK(cudaStreamSynchronize(s));
  *n = (int32_t)std::min<unsigned>(cnt, (unsigned)kTraceCap);
  return OCRDEC_OK;
}

int ocrdec_replay_moe_ffn(ocrdec_ctx* c, int batch, int k, int first_layer, int n_layers, ocrdec_stream stream) {
  int st = check_ready(c);
  if (st) return st;
  if ((st = check_bk(c, batch, k))) return st;
  const ocrdec_config& m = c->cfg;
  if (first_layer < m.n_dense_first || n_layers < 1 || first_layer + n_layers > m.n_layers) return OCRDEC_EINVAL;
  const LaunchCfg lc = c->lc(reinterpret_cast<cudaStream_t>(stream));
  // the same launches (row bound batch * (k + 1)) as the verify pass of a step
  for (int l = first_layer; l < first_layer + n_layers; ++l) {
    st = moe_ffn(c, lc, batch * (k + 1), c->layers[l], true);
    if (st) return st;
  }
  return OCRDEC_OK;
}

size_t ocrdec_draft_head_fp8_bytes(const ocrdec_config* cfg) {
  if (!config_ok(cfg)) return 0;
  return align_up((size_t)cfg->vocab * cfg->d_model) + (size_t)cfg->vocab * sizeof(float);
}

int ocrdec_set_draft_head_fp8(ocrdec_ctx* c, void* buf, size_t bytes, ocrdec_stream stream) {
  if (!c) return OCRDEC_EINVAL;
  if (!buf) {
    c->head8 = nullptr;
    c->head8_inv = nullptr;
    c->drop_graphs();
    return OCRDEC_OK;
  }
  if (!c->have_weights) return OCRDEC_ESTATE;
  const ocrdec_config& m = c->cfg;
  if ((reinterpret_cast<uintptr_t>(buf) & 255) || bytes < ocrdec_draft_head_fp8_bytes(&m)) return OCRDEC_EINVAL;
  if (m.d_model % (2 * kChunk)) return OCRDEC_EINVAL;  // whole 128-byte rows of e4m3 pairs
  unsigned char* w8 = static_cast<unsigned char*>(buf);
  float* inv = reinterpret_cast<float*>(w8 + align_up((size_t)m.vocab * m.d_model));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  quantize_rows_e4m3_kernel<<<(m.vocab + 7) / 8, 256, 0, s>>>(c->lm_head.p, m.vocab, m.d_model, w8, inv);
  CK(cudaGetLastError());
  // the e4m3 matrix read as [V][d/2] byte pairs: the bf16 tiles' geometry
  CK(encode_weight_map(w8, m.d_model / 2, m.vocab, 1, &c->head8_map));
  c->head8 = w8;
  c->head8_inv = inv;
  c->drop_graphs();
  return OCRDEC_OK;
}

int ocrdec_set_draft_taps(ocrdec_ctx* c, float* logits) {
  if (!c) return OCRDEC_EINVAL;
  c->dbg_draft_logits = logits;
  c->drop_graphs();
  return OCRDEC_OK;
}

int ocrdec_set_debug_taps(ocrdec_ctx* c, float* hidden, float* logits) {
  if (!c) return OCRDEC_EINVAL;
  c->dbg_hidden = hidden;
  c->dbg_logits = logits;
  c->drop_graphs();
  return OCRDEC_OK;
}

const char* ocrdec_strerror(int s) {
  switch (s) {
    case OCRDEC_OK: return "ok";
    case OCRDEC_EINVAL: return "invalid argument";
    case OCRDEC_ENOMEM: return "workspace too small";
    case OCRDEC_ECUDA: return "CUDA runtime error";
    case OCRDEC_ECAPACITY: return "KV capacity exceeded";
    case OCRDEC_ETIMEOUT: return "device wait timed out";
    case OCRDEC_ESTATE: return "call order violated";
    default: return "unknown status";
  }
}

// ---- single-kernel entry points -------------------------------------------

size_t ocrdec_op_scratch_bytes(void) {
  int sms = device_sms();
  return op_scratch_layout(sms > 0 ? sms : 148, nullptr, nullptr, nullptr);
}

int ocrdec_op_norm_gemv(const void* W, const float* x, const void* g, float eps, int R, int N, int K, float* y,
                        void* scratch, ocrdec_stream stream) {
  if (!W || !x || !g || !y || !scratch || R < 1 || R > kRmax || N < 1 || K < kChunk || K % kChunk || K > kGemvMaxK)
    return OCRDEC_EINVAL;
  if ((reinterpret_cast<uintptr_t>(W) & 15) || (reinterpret_cast<uintptr_t>(scratch) & 255)) return OCRDEC_EINVAL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* st = static_cast<int*>(scratch);
  CK(prepare_kernels());
  const int sms = device_sms();
  size_t am_off, ctr_off, part_off;
  op_scratch_layout(sms, &am_off, &ctr_off, &part_off);
  CK(cudaMemsetAsync(st, 0, part_off, s));  // status, counters, tile counters
  GemvLaunch gl;
  CK(encode_weight_map(W, K, N, 1, &gl.tm_w));
  gl.s.N = N;
  gl.s.K = K;
  gl.s.rows_static = R;
  gl.s.status = st;
  gemv_plan(gl.s);
  gl.s.kparts = gemv_kparts(gl.s, 2 * sms);
  gl.s.part = reinterpret_cast<float*>(static_cast<char*>(scratch) + part_off);
  gl.s.tile_counter = reinterpret_cast<int*>(static_cast<char*>(scratch) + ctr_off);
  gl.s.work = st + 12;
  gl.src = SrcKind::Norm;
  gl.norm = SrcNorm::Params{x, K, nullptr, static_cast<const bf16*>(g), eps};
  gl.epi = EpiKind::Store;
  gl.store = EpiStore<false>::Params{y, N, 1, nullptr};
  gl.rows_bound = R;
  LaunchCfg lc{s, false, sms};
  CK(launch_gemv(gl, lc));
  return OCRDEC_OK;
}

int ocrdec_op_lm_argmax(const void* W, const float* x, const void* g, float eps, int R, int N, int K, int32_t* tok,
                        float* logits, void* scratch, ocrdec_stream stream) {
  if (!W || !x || !g || !tok || !scratch || R < 1 || R > kRmax || N < 1 || K < kChunk || K % kChunk || K > kGemvMaxK)
    return OCRDEC_EINVAL;
  if ((reinterpret_cast<uintptr_t>(W) & 15) || (reinterpret_cast<uintptr_t>(scratch) & 255)) return OCRDEC_EINVAL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* st = static_cast<int*>(scratch);
  CK(prepare_kernels());
  const int sms = device_sms();
  size_t am_off;
  op_scratch_layout(sms, &am_off, nullptr, nullptr);
  CK(cudaMemsetAsync(st, 0, 64, s));  // status, trace header (off), counter
  GemvLaunch gl;
  CK(encode_weight_map(W, K, N, 1, &gl.tm_w));
  gl.s.N = N;
  gl.s.K = K;
  gl.s.rows_static = R;
  gl.s.status = st;
  gl.s.counter = st + 8;  // clear of the trace header (st[1], st[2])
  gl.s.work = st + 12;
  gemv_plan(gl.s);
  gl.src = SrcKind::Norm;
  gl.norm = SrcNorm::Params{x, K, nullptr, static_cast<const bf16*>(g), eps};
  gl.epi = EpiKind::Argmax;
  gl.argmax = EpiArgmax::Params{tok, 1, logits, reinterpret_cast<float2*>(static_cast<char*>(scratch) + am_off), nullptr};
  gl.rows_bound = R;
  gl.grid = std::min(gl.s.tiles_per_mat, 2 * sms);
  LaunchCfg lc{s, false, sms};
  CK(launch_gemv(gl, lc));
  return OCRDEC_OK;
}

}  // extern "C"

// ---- LM-head argmax on library-owned scratch ---------------------------------
// Fixed scratch in the library's own device image, one copy per device.  Its
// address is looked up once per device (cudaGetSymbolAddress) by the first
// call made with that device current; later calls reuse it.  Nothing here
// allocates device memory.
namespace {
constexpr size_t kStaticScratchBytes = 64 << 10;
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];
constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices] = {};
}  // namespace

extern "C" {

size_t ocrdec_op_static_scratch_bytes(void) { return kStaticScratchBytes; }

int ocrdec_op_lm_argmax_static(const void* W, const float* x, const void* g, float eps, int R, int N, int K,
                               int32_t* tok, float* logits, ocrdec_stream stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return OCRDEC_ECUDA;
  const int sms = device_sms();
  if (sms <= 0) return OCRDEC_ECUDA;
  size_t am_off;
  op_scratch_layout(sms, &am_off, nullptr, nullptr);
  // status words + one (value, index) partial per CTA and row; the CTA count is
  // at most two per SM
  if (am_off + sizeof(float2) * 2 * (size_t)sms * kRmax > kStaticScratchBytes) return OCRDEC_ENOMEM;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return OCRDEC_ECUDA;
      g_static_ptr[dev] = p;
    }
    scratch = g_static_ptr[dev];
  }
  return ocrdec_op_lm_argmax(W, x, g, eps, R, N, K, tok, logits, scratch, stream);
}

}  // extern "C"
