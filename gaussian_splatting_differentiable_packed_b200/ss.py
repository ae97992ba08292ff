"""ctypes binding of libss.so (include/ss.h) — argument marshalling only.

Every function here forwards torch CUDA tensors' device pointers and the
current CUDA stream to the C entry point of the same name and raises SSError
on a non-zero status.  No step of the splatting path runs in Python or on the
CPU: if libss.so is missing the import of the library fails loudly.
PyTorch only allocates device memory and provides the stream.

`PackedStep` strings the calls into one forward+backward step with buffers
owned by torch (the counts returned by the two synchronising calls size the
later buffers; capacities grow with headroom when exceeded).  Around it:
`HostPipeline` (steps over pinned host inputs and gradients, copies
overlapped with the kernels), `AdamTrainer` (the projection backward fused
with Adam) and `GradQuantAccum` (16-bit block-quantised gradient
accumulators for ss_project_bwd_gq).
"""
from __future__ import annotations

import ctypes as ct
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libss.so")

SS_OK, SS_ERR_INVALID_ARG, SS_ERR_CAPACITY, SS_ERR_OVERFLOW, SS_ERR_CUDA, SS_ERR_DEVICE_CHECK = range(6)
SIZE_MASK_WORDS, SIZE_MASK_BLOCKS, SIZE_TILES_X, SIZE_TILES_Y, SIZE_N_TILES, SIZE_N_PAD = range(6)
WS_PROJECT, WS_INTERSECT, WS_SORT, WS_TILE_ORDER = range(4)
ROW = 12
PMASK_BLOCK = 128
TILE = 16

EXPORTS = ("ss_size", "ss_workspace_bytes", "ss_status_string", "ss_last_error", "ss_project_packed",
           "ss_intersect_tiles", "ss_sort_isects", "ss_sort_isects_noalloc", "ss_tile_order", "ss_rasterize_fwd",
           "ss_rasterize_fwd_counts",
           "ss_rasterize_bwd", "ss_project_bwd", "ss_project_bwd_adam", "ss_project_bwd_gq")


class ss_adam(ct.Structure):
    _fields_ = [("lr_means", ct.c_float), ("lr_quats", ct.c_float), ("lr_scales", ct.c_float),
                ("lr_opacities", ct.c_float), ("lr_sh_dc", ct.c_float), ("lr_sh_rest", ct.c_float),
                ("beta1", ct.c_float), ("beta2", ct.c_float), ("eps", ct.c_float), ("step", ct.c_int32)]


class ss_adam_state(ct.Structure):
    _fields_ = [(n, ct.c_void_p) for n in ("m_means", "v_means", "m_quats", "v_quats", "m_scales", "v_scales",
                                           "m_opacities", "v_opacities", "m_sh", "v_sh")]


class ss_gq_accum(ct.Structure):
    _fields_ = [(n, ct.c_void_p) for n in ("means", "quats", "scales", "opacities", "sh_dc", "sh_rest",
                                           "block_scale")]


class ss_dims(ct.Structure):
    _fields_ = [("C", ct.c_int32), ("W", ct.c_int32), ("H", ct.c_int32), ("sh_degree", ct.c_int32),
                ("N", ct.c_int64), ("near_plane", ct.c_float), ("far_plane", ct.c_float)]


class SSError(RuntimeError):
    def __init__(self, status: int, call: str, msg: str, count: int | None = None):
        super().__init__(f"{call}: {msg} (status {status})")
        self.status = status
        self.count = count


_lib = None


def lib() -> ct.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m gaussian_splatting_differentiable_packed_b200.build`")
        L = ct.CDLL(LIB_PATH)
        P, i64, i32, sz = ct.c_void_p, ct.c_int64, ct.c_int, ct.c_size_t
        D = ct.POINTER(ss_dims)
        L.ss_size.argtypes = [D, i32]
        L.ss_size.restype = i64
        L.ss_workspace_bytes.argtypes = [D, i32, i64]
        L.ss_workspace_bytes.restype = sz
        L.ss_status_string.argtypes = [i32]
        L.ss_status_string.restype = ct.c_char_p
        L.ss_last_error.argtypes = []
        L.ss_last_error.restype = ct.c_char_p
        L.ss_project_packed.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, P, i64, i64, P, sz, ct.POINTER(i64), P]
        L.ss_intersect_tiles.argtypes = [D, P, P, P, i64, P, P, P, P, i64, P, sz, ct.POINTER(ct.c_uint64), P]
        L.ss_sort_isects.argtypes = [D, P, P, P, P, i64, i32, P, P, sz, P, ct.POINTER(i32), P]
        L.ss_sort_isects_noalloc.argtypes = [D, P, P, P, P, i64, P, ct.POINTER(i32), P]
        L.ss_tile_order.argtypes = [D, P, P, P, sz, P]
        L.ss_rasterize_fwd.argtypes = [D, P, P, P, P, P, P, P, P, P, P]
        L.ss_rasterize_fwd_counts.argtypes = [D, P, P, P, P, P, P, P, P]
        L.ss_rasterize_bwd.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, i64, P]
        L.ss_project_bwd.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P]
        L.ss_project_bwd_adam.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, ct.POINTER(ss_adam_state),
                                          ct.POINTER(ss_adam), P]
        L.ss_project_bwd_gq.argtypes = [D, P, P, P, P, P, P, P, P, P, ct.POINTER(ss_gq_accum), i32, P]
        for f in ("ss_project_packed", "ss_intersect_tiles", "ss_sort_isects", "ss_sort_isects_noalloc",
                  "ss_tile_order", "ss_rasterize_fwd",
                  "ss_rasterize_fwd_counts", "ss_rasterize_bwd", "ss_project_bwd", "ss_project_bwd_adam",
                  "ss_project_bwd_gq"):
            getattr(L, f).restype = i32
        _lib = L
    return _lib


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ct.c_void_p(t)
    return ct.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ct.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ct.c_void_p(stream)
    return ct.c_void_p(stream.cuda_stream)


def _check(status: int, call: str, count=None):
    if status != SS_OK:
        msg = lib().ss_last_error().decode() or lib().ss_status_string(status).decode()
        raise SSError(status, call, msg, count)


def make_dims(C, W, H, sh_degree, N, near=0.01, far=1e10) -> ss_dims:
    return ss_dims(C, W, H, sh_degree, N, near, far)


def size(d: ss_dims, what: int) -> int:
    v = lib().ss_size(ct.byref(d), what)
    if v < 0:
        raise SSError(SS_ERR_INVALID_ARG, "ss_size", "invalid dims")
    return int(v)


def workspace_bytes(d: ss_dims, which: int, count: int = 0) -> int:
    return int(lib().ss_workspace_bytes(ct.byref(d), which, count))


def ss_project_packed(d, cams, means, quats, scales, opacities, sh, mask, block_count, block_off, screen, aabb16,
                      row_depth, cap_rows, temp, stream=None, cap_visible=None) -> int:
    """cap_visible: the per-image visible cap (None: no cap)."""
    nnz = ct.c_int64(0)
    st = lib().ss_project_packed(ct.byref(d), _p(cams), _p(means), _p(quats), _p(scales), _p(opacities), _p(sh),
                                 _p(mask), _p(block_count), _p(block_off), _p(screen), _p(aabb16), _p(row_depth),
                                 int(cap_rows), -1 if cap_visible is None else int(cap_visible),
                                 _p(temp), 0 if temp is None else temp.numel() * temp.element_size(),
                                 ct.byref(nnz), _stream(stream))
    _check(st, "ss_project_packed", int(nnz.value))
    return int(nnz.value)


def ss_intersect_tiles(d, row_depth, aabb16, block_off, nnz, isect_off, keys, vals, cap_isects, temp,
                       stream=None, key_hist=None) -> int:
    """key_hist: optional device uint32 [4*256], set to the digit counts of
    the keys' tile-id bytes (for ss_sort_isects)."""
    n = ct.c_uint64(0)
    st = lib().ss_intersect_tiles(ct.byref(d), _p(row_depth), _p(aabb16), _p(block_off), int(nnz), _p(isect_off),
                                  _p(keys), _p(vals), _p(key_hist), int(cap_isects), _p(temp),
                                  0 if temp is None else temp.numel() * temp.element_size(), ct.byref(n),
                                  _stream(stream))
    _check(st, "ss_intersect_tiles", int(n.value))
    return int(n.value)


def ss_sort_isects(d, keys_a, vals_a, keys_b, vals_b, n, temp, tile_off, stream=None, presorted_depth=False,
                   key_hist=None) -> bool:
    """presorted_depth: the keys arrive in depth order (as ss_intersect_tiles
    writes them), so only the tile-id bytes are sorted; key_hist: their digit
    counts as ss_intersect_tiles wrote them (skips the histogram read)."""
    in_b = ct.c_int(0)
    st = lib().ss_sort_isects(ct.byref(d), _p(keys_a), _p(vals_a), _p(keys_b), _p(vals_b), int(n),
                              1 if presorted_depth else 0, _p(key_hist), _p(temp),
                              0 if temp is None else temp.numel() * temp.element_size(), _p(tile_off),
                              ct.byref(in_b), _stream(stream))
    _check(st, "ss_sort_isects")
    return bool(in_b.value)


def ss_sort_isects_noalloc(d, keys_a, vals_a, keys_b, vals_b, n, tile_off, stream=None) -> bool:
    """ss_sort_isects with the library's static scratch (no caller temp buffer)."""
    in_b = ct.c_int(0)
    st = lib().ss_sort_isects_noalloc(ct.byref(d), _p(keys_a), _p(vals_a), _p(keys_b), _p(vals_b), int(n),
                                      _p(tile_off), ct.byref(in_b), _stream(stream))
    _check(st, "ss_sort_isects_noalloc")
    return bool(in_b.value)


def ss_tile_order(d, tile_off, tile_order, temp, stream=None):
    _check(lib().ss_tile_order(ct.byref(d), _p(tile_off), _p(tile_order), _p(temp),
                               0 if temp is None else temp.numel() * temp.element_size(), _stream(stream)),
           "ss_tile_order")


def ss_rasterize_fwd(d, screen, vals, tile_off, img, T_final, last_id, depth=None, bg=None, stream=None,
                     tile_order=None):
    _check(lib().ss_rasterize_fwd(ct.byref(d), _p(screen), _p(vals), _p(tile_off), _p(tile_order), _p(img),
                                  _p(T_final), _p(last_id), _p(depth), _p(bg), _stream(stream)), "ss_rasterize_fwd")


def ss_rasterize_fwd_counts(d, screen, vals, tile_off, img, T_final, last_id, counts, stream=None):
    _check(lib().ss_rasterize_fwd_counts(ct.byref(d), _p(screen), _p(vals), _p(tile_off), _p(img), _p(T_final),
                                         _p(last_id), _p(counts), _stream(stream)), "ss_rasterize_fwd_counts")


def raster_work(d, step) -> dict:
    """Exact per-launch work counts of the rasterizers for the step's last
    forward (runs the counting forward once; not part of any timed region)."""
    counts = torch.zeros(5, dtype=torch.int64, device=step.dev)
    ss_rasterize_fwd_counts(d, step.screen, step.vals, step.tile_off, step.img, step.T, step.last, counts)
    c = [int(x) for x in counts.cpu().tolist()]
    return dict(evals=c[0], exps=c[1], comps=c[2], bwd_evals=c[3], bwd_exps=c[4])


def ss_rasterize_bwd(d, screen, vals, tile_off, T_final, last_id, v_img, v_T, v_screen, nnz, stream=None,
                     v_depth=None, bg=None, tile_order=None):
    _check(lib().ss_rasterize_bwd(ct.byref(d), _p(screen), _p(vals), _p(tile_off), _p(tile_order), _p(T_final),
                                  _p(last_id), _p(v_img), _p(v_T), _p(v_depth), _p(bg), _p(v_screen), int(nnz),
                                  _stream(stream)),
           "ss_rasterize_bwd")


def ss_project_bwd(d, cams, means, quats, scales, opacities, sh, mask, block_off, v_screen, v_means, v_quats,
                   v_scales, v_opacities, v_sh, stream=None):
    _check(lib().ss_project_bwd(ct.byref(d), _p(cams), _p(means), _p(quats), _p(scales), _p(opacities), _p(sh),
                                _p(mask), _p(block_off), _p(v_screen), _p(v_means), _p(v_quats), _p(v_scales),
                                _p(v_opacities), _p(v_sh), _stream(stream)), "ss_project_bwd")


def ss_project_bwd_adam(d, cams, means, quats, log_scales, scales, logit_opacities, opacities, sh, mask, block_off,
                        v_screen, state: dict, hp: ss_adam, stream=None):
    """Fused projection backward + Adam.  state maps m_/v_ + (means, quats,
    scales, opacities, sh) to device tensors shaped like the parameters."""
    st = ss_adam_state(*[_p(state[n]) for n, _ in ss_adam_state._fields_])
    _check(lib().ss_project_bwd_adam(ct.byref(d), _p(cams), _p(means), _p(quats), _p(log_scales), _p(scales),
                                     _p(logit_opacities), _p(opacities), _p(sh), _p(mask), _p(block_off),
                                     _p(v_screen), ct.byref(st), ct.byref(hp), _stream(stream)),
           "ss_project_bwd_adam")


GQ_BLOCK = 256
GQ_ATTRS = ("means", "quats", "scales", "opacities", "sh_dc", "sh_rest")


class GradQuantAccum:
    """Block-quantised gradient accumulators of N Gaussians (ss_project_bwd_gq):
    int16 codes per attribute and the [6, ceil(N/256)] block scales, on the
    device.  decoded() gives the accumulated values (code * block scale) for
    inspection; the step itself never decodes outside the kernel."""

    def __init__(self, N: int, K: int, device="cuda"):
        self.N, self.K = int(N), int(K)
        widths = dict(means=3, quats=4, scales=3, opacities=1, sh_dc=3, sh_rest=3 * (self.K - 1))
        dev = torch.device(device)
        self.codes = {a: torch.zeros((self.N, max(w, 1)), dtype=torch.int16, device=dev) for a, w in widths.items()}
        self.widths = widths
        self.nb = (self.N + GQ_BLOCK - 1) // GQ_BLOCK
        self.block_scale = torch.zeros((len(GQ_ATTRS), max(self.nb, 1)), dtype=torch.float32, device=dev)

    def struct(self) -> ss_gq_accum:
        ptr = [_p(self.codes[a]) if self.widths[a] > 0 else None for a in GQ_ATTRS]
        return ss_gq_accum(*ptr, _p(self.block_scale))

    def decoded(self) -> dict:
        out = {}
        for i, a in enumerate(GQ_ATTRS):
            per_row = self.block_scale[i].repeat_interleave(GQ_BLOCK)[: self.N].double().unsqueeze(1)
            out[a] = (self.codes[a][:, : self.widths[a]].double() * per_row).cpu().numpy()
        return out


def ss_project_bwd_gq(d, cams, means, quats, scales, opacities, sh, mask, block_off, v_screen,
                      acc: GradQuantAccum, first: bool, stream=None):
    """Projection backward that adds its gradients into block-quantised
    accumulators (first=True starts them from zero)."""
    st = acc.struct()
    _check(lib().ss_project_bwd_gq(ct.byref(d), _p(cams), _p(means), _p(quats), _p(scales), _p(opacities), _p(sh),
                                   _p(mask), _p(block_off), _p(v_screen), ct.byref(st), 1 if first else 0,
                                   _stream(stream)),
           "ss_project_bwd_gq")


class AdamTrainer:
    """Training steps on one PackedStep with the fused projection backward +
    Adam: the parameters (means, raw quats, log-scales, logit-opacities, SH),
    their activated copies and the moments live on the device and are updated
    in place each step; no gradient arrays are written.

    step(v_img_fn) runs forward, the rasterizer backward with the upstream
    gradient v_img_fn(img) and the fused update, and returns the image."""

    def __init__(self, step: "PackedStep", cams, means, quats, log_scales, logit_opacities, sh,
                 lr=(1.6e-4, 1e-3, 5e-3, 5e-2, 2.5e-3, 1.25e-4), beta1=0.9, beta2=0.999, eps=1e-15):
        self.step_obj = step
        self.cams, self.means, self.quats, self.sh = cams, means, quats, sh
        self.log_scales, self.logit_opacities = log_scales, logit_opacities
        self.scales = torch.exp(log_scales).contiguous()
        self.opacities = torch.sigmoid(logit_opacities).contiguous()
        self.state = {}
        for name, ref in (("means", means), ("quats", quats), ("scales", log_scales),
                          ("opacities", logit_opacities), ("sh", sh)):
            self.state["m_" + name] = torch.zeros_like(ref)
            self.state["v_" + name] = torch.zeros_like(ref)
        self.hp = ss_adam(*lr, beta1, beta2, eps, 0)

    def step(self, v_img_fn, stream=None):
        s = self.step_obj
        img = s.forward(self.cams, self.means, self.quats, self.scales, self.opacities, self.sh, stream)
        v_img = v_img_fn(img)
        ss_rasterize_bwd(s.d, s.screen, s.vals, s.tile_off, s.T, s.last, v_img, None, s.v_screen, s.nnz, stream,
                         tile_order=s.tile_order)
        self.hp.step += 1
        ss_project_bwd_adam(s.d, self.cams, self.means, self.quats, self.log_scales, self.scales,
                            self.logit_opacities, self.opacities, self.sh, s.mask, s.block_off, s.v_screen,
                            self.state, self.hp, stream)
        return img


def _u32(n, dev):
    return torch.empty(max(int(n), 1), dtype=torch.int32, device=dev)


class PackedStep:
    """One forward+backward step over fixed dims, buffers owned by torch.

    forward() runs ss_project_packed, ss_intersect_tiles, ss_sort_isects,
    ss_tile_order and ss_rasterize_fwd; backward(v_img, v_T=None) runs ss_rasterize_bwd and
    ss_project_bwd.  forward(..., bg=, depth=True) also blends a background
    colour per camera and renders the expected depth (self.depth);
    backward(..., v_depth=) then takes its gradient.  cap_visible applies the
    per-image visible cap of ss_project_packed (None: no cap).  Intermediate
    buffers are kept as attributes so callers (tests) can inspect every stage.
    """

    def __init__(self, d: ss_dims, device="cuda", cap_rows: int = 0, cap_isects: int = 0, headroom: float = 1.25,
                 cap_visible: int | None = None):
        self.d = d
        self.cap_visible = cap_visible
        self.dev = torch.device(device)
        self.headroom = headroom
        C, N = d.C, d.N
        self.K = (d.sh_degree + 1) ** 2
        self.mask_words = size(d, SIZE_MASK_WORDS)
        self.mask_blocks = size(d, SIZE_MASK_BLOCKS)
        self.n_tiles = size(d, SIZE_N_TILES)
        dev = self.dev
        self.mask = _u32(self.mask_words, dev)
        self.block_count = _u32(self.mask_blocks, dev)
        self.block_off = torch.empty(self.mask_blocks + 1, dtype=torch.int64, device=dev)
        self.temp_project = torch.empty(workspace_bytes(d, WS_PROJECT), dtype=torch.uint8, device=dev)
        self.tile_off = torch.empty(self.n_tiles + 1, dtype=torch.int64, device=dev)
        self.key_hist = torch.empty(4 * 256, dtype=torch.int32, device=dev)  # digit counts of the keys' tile ids
        self.tile_order = _u32(self.n_tiles, dev)
        self.temp_order = torch.empty(workspace_bytes(d, WS_TILE_ORDER), dtype=torch.uint8, device=dev)
        self.img = torch.empty((C, d.H, d.W, 3), dtype=torch.float32, device=dev)
        self.T = torch.empty((C, d.H, d.W), dtype=torch.float32, device=dev)
        self.last = torch.empty((C, d.H, d.W), dtype=torch.int32, device=dev)
        self.v_means = torch.empty((N, 3), dtype=torch.float32, device=dev)
        self.v_quats = torch.empty((N, 4), dtype=torch.float32, device=dev)
        self.v_scales = torch.empty((N, 3), dtype=torch.float32, device=dev)
        self.v_opacities = torch.empty((N,), dtype=torch.float32, device=dev)
        self.v_sh = torch.empty((N, self.K, 3), dtype=torch.float32, device=dev)
        self.cap_rows = 0
        self.cap_isects = 0
        self._rows(cap_rows)
        self._isects(cap_isects)
        self.nnz = 0
        self.n_isects = 0
        self.result_in_b = False

    def _rows(self, cap):
        cap = max(int(cap), 1)
        if cap <= self.cap_rows:
            return
        dev = self.dev
        self.screen = torch.empty((cap, ROW), dtype=torch.float32, device=dev)
        self.aabb16 = torch.empty((cap, 2), dtype=torch.int32, device=dev)
        self.row_depth = torch.empty(cap, dtype=torch.float32, device=dev)
        self.isect_off = torch.empty(cap + 1, dtype=torch.int64, device=dev)
        self.v_screen = torch.empty((cap, ROW), dtype=torch.float32, device=dev)
        self.temp_isect = torch.empty(workspace_bytes(self.d, WS_INTERSECT, cap), dtype=torch.uint8, device=dev)
        self.cap_rows = cap

    def _isects(self, cap):
        cap = max(int(cap), 1)
        if cap <= self.cap_isects:
            return
        dev = self.dev
        self.keys_a = torch.empty(cap, dtype=torch.int64, device=dev)
        self.vals_a = torch.empty(cap, dtype=torch.int32, device=dev)
        self.keys_b = torch.empty(cap, dtype=torch.int64, device=dev)
        self.vals_b = torch.empty(cap, dtype=torch.int32, device=dev)
        self.temp_sort = torch.empty(workspace_bytes(self.d, WS_SORT, cap), dtype=torch.uint8, device=dev)
        self.cap_isects = cap

    def forward(self, cams, means, quats, scales, opacities, sh, stream=None, bg=None, depth=False):
        self.inputs = (cams, means, quats, scales, opacities, sh)
        self.bg = bg
        d = self.d
        try:
            nnz = ss_project_packed(d, cams, means, quats, scales, opacities, sh, self.mask, self.block_count,
                                    self.block_off, self.screen, self.aabb16, self.row_depth, self.cap_rows,
                                    self.temp_project, stream, cap_visible=self.cap_visible)
        except SSError as e:
            if e.status != SS_ERR_CAPACITY:
                raise
            self._rows(int(e.count * self.headroom) + 1)
            nnz = ss_project_packed(d, cams, means, quats, scales, opacities, sh, self.mask, self.block_count,
                                    self.block_off, self.screen, self.aabb16, self.row_depth, self.cap_rows,
                                    self.temp_project, stream, cap_visible=self.cap_visible)
        self.nnz = nnz
        try:
            n = ss_intersect_tiles(d, self.row_depth, self.aabb16, self.block_off, nnz, self.isect_off,
                                   self.keys_a, self.vals_a, self.cap_isects, self.temp_isect, stream,
                                   key_hist=self.key_hist)
        except SSError as e:
            if e.status != SS_ERR_CAPACITY:
                raise
            self._isects(int(e.count * self.headroom) + 1)
            n = ss_intersect_tiles(d, self.row_depth, self.aabb16, self.block_off, nnz, self.isect_off,
                                   self.keys_a, self.vals_a, self.cap_isects, self.temp_isect, stream,
                                   key_hist=self.key_hist)
        self.n_isects = n
        self.unsorted_keys = self.keys_a
        self.unsorted_vals = self.vals_a
        self.result_in_b = ss_sort_isects(d, self.keys_a, self.vals_a, self.keys_b, self.vals_b, n, self.temp_sort,
                                          self.tile_off, stream, presorted_depth=True, key_hist=self.key_hist)
        self.keys = self.keys_b if self.result_in_b else self.keys_a
        self.vals = self.vals_b if self.result_in_b else self.vals_a
        ss_tile_order(d, self.tile_off, self.tile_order, self.temp_order, stream)
        if depth and getattr(self, "depth", None) is None:
            self.depth = torch.empty((d.C, d.H, d.W), dtype=torch.float32, device=self.dev)
        ss_rasterize_fwd(d, self.screen, self.vals, self.tile_off, self.img, self.T, self.last,
                         self.depth if depth else None, bg, stream, tile_order=self.tile_order)
        return self.img

    def backward(self, v_img, v_T=None, stream=None, v_depth=None):
        cams, means, quats, scales, opacities, sh = self.inputs
        d = self.d
        ss_rasterize_bwd(d, self.screen, self.vals, self.tile_off, self.T, self.last, v_img, v_T, self.v_screen,
                         self.nnz, stream, v_depth=v_depth, bg=self.bg, tile_order=self.tile_order)
        ss_project_bwd(d, cams, means, quats, scales, opacities, sh, self.mask, self.block_off, self.v_screen,
                       self.v_means, self.v_quats, self.v_scales, self.v_opacities, self.v_sh, stream)
        return dict(v_means=self.v_means, v_quats=self.v_quats, v_scales=self.v_scales,
                    v_opacities=self.v_opacities, v_sh=self.v_sh)


def scene_tensors(scene, device="cuda"):
    """Device copies of a scenes.Scene's inputs (cams, means, quats, scales, opacities, sh)."""
    f = lambda a: torch.from_numpy(a).to(device=device, dtype=torch.float32).contiguous()
    return (f(scene.cams), f(scene.means), f(scene.quats), f(scene.scales), f(scene.opacities), f(scene.sh))


def scene_dims(scene) -> ss_dims:
    return make_dims(scene.C, scene.W, scene.H, scene.sh_degree, scene.N, scene.near, scene.far)


def _varying_bytes(k, shifts) -> int:
    n = 0
    for sh in shifts:
        dig = (k >> sh) & 0xFF
        n += int(dig.min().item()) != int(dig.max().item())
    return n


def sort_passes_for(keys, d: ss_dims, presorted_depth: bool = True) -> int:
    """Digit passes ss_sort_isects runs on these (unsorted or sorted) keys:
    one per byte the tile ids need and, unless the keys arrive in depth order,
    per byte of the depth, less the bytes that are equal in every key.
    Measurement helper (torch reductions); not part of any step."""
    if keys.numel() == 0:
        return 0
    k = keys.to(torch.int64)
    tb = max(0, (size(d, SIZE_N_TILES) - 1).bit_length())
    hi = [32 + 8 * i for i in range(max((tb + 7) // 8, 1 if presorted_depth else 0))]
    return _varying_bytes(k, ([] if presorted_depth else [0, 8, 16, 24]) + hi)


def depth_sort_passes(row_depth) -> int:
    """Digit passes of the intersection's depth sort of its rows: the bytes of
    the rows' depth bits that are not equal in every row.  Measurement helper."""
    if row_depth.numel() == 0:
        return 0
    return _varying_bytes(row_depth.view(torch.int32).to(torch.int64) & 0xFFFFFFFF, [0, 8, 16, 24])


def seen_gaussians(d: ss_dims, mask) -> int:
    """Gaussians that some camera sees (a set bit in one of their mask words).
    Measurement helper (torch reductions); not part of any step."""
    words = size(d, SIZE_MASK_WORDS) // d.C
    m = mask[: d.C * words].view(d.C, words)
    u = m[0].clone()
    for c in range(1, d.C):
        u |= m[c]
    b = u.view(torch.uint8).to(torch.int32)
    pop = torch.zeros_like(b)
    for k in range(8):
        pop += (b >> k) & 1
    return int(pop.sum().item())


def sort_launches(n_isects: int, passes: int, given_hist: bool = True) -> int:
    """Kernels of one ss_sort_isects call: histogram (none when the digit
    counts come with the keys), digit bases, one onesweep kernel per digit
    pass that runs, tile ranges (the runs' first keys after the last pass, or
    every key when no pass runs)."""
    return 0 if n_isects == 0 else (2 if given_hist else 3) + passes


def launches_per_step(d: ss_dims, nnz: int, n_isects: int, sort_passes: int, depth_passes: int) -> int:
    """Kernels libss launches in one forward+backward step (memsets excluded):
    projection 5 (pass 1, three scan kernels, pass 2), intersection 3 plus
    one per depth-sort pass (row depth keys with the count and the depth
    bytes' digit counts, the depth sort's bases, the fused offsets-and-write
    kernel), the sort
    (sort_launches), tile order 3 (histogram, scan, scatter), rasterizer
    1 + 1, projection backward 1.  With no Gaussians only the tile order and
    the two rasterizers launch (they still write the empty images)."""
    if d.N == 0:
        return 3 + 2
    n = 5
    if nnz > 0:
        n += 3 + depth_passes
    n += sort_launches(n_isects, sort_passes)
    return n + 3 + 3


class HostPipeline:
    """PackedStep steps over inputs and gradients that live in pinned host
    memory, with the transfers overlapped: while step k's kernels run on the
    compute stream, step k+1's inputs go host -> device on one copy stream and
    step k-1's gradients go device -> host on another.  Device inputs and
    gradient outputs are double-buffered (2 x parameters + 2 x gradients of
    device memory); events order every reuse of a buffer.

    run(host_steps) takes a list of (inputs, v_img, outputs) per step: inputs
    are the six pinned host tensors of PackedStep.forward, v_img the pinned
    upstream gradient, outputs a dict of pinned host tensors named like the
    gradients (v_means, v_quats, v_scales, v_opacities, v_sh) that receive the
    step's gradients.  Returns an event recorded after the last gradient
    copy (on the copy stream) once everything has been enqueued; synchronize
    on it (or call sync()) before reading the outputs.  With start (an event
    recorded on the compute stream) the first upload waits for it, so a timed
    region bracketed by start and the returned event holds every copy.
    """

    GRADS = ("v_means", "v_quats", "v_scales", "v_opacities", "v_sh")

    def __init__(self, step: "PackedStep", example_inputs, example_v_img):
        self.step = step
        dev = step.dev
        self.compute = torch.cuda.current_stream(dev)
        self.up = torch.cuda.Stream(dev)
        self.down = torch.cuda.Stream(dev)
        self.dev_in = [[torch.empty(t.shape, dtype=t.dtype, device=dev) for t in example_inputs] for _ in range(2)]
        self.dev_vimg = [torch.empty(example_v_img.shape, dtype=example_v_img.dtype, device=dev) for _ in range(2)]
        self.dev_out = [{k: torch.empty_like(getattr(step, k)) for k in self.GRADS} for _ in range(2)]
        self.in_free = [None, None]   # compute finished reading buffer p
        self.out_free = [None, None]  # device -> host copy of buffer p finished

    def _upload(self, k, inputs, v_img, after=None):
        p = k % 2
        ev = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.up):
            if after is not None:
                self.up.wait_event(after)
            if self.in_free[p] is not None:
                self.up.wait_event(self.in_free[p])
            for dst, src in zip(self.dev_in[p], inputs):
                dst.copy_(src, non_blocking=True)
            self.dev_vimg[p].copy_(v_img, non_blocking=True)
            ev.record(self.up)
        return ev

    def run(self, host_steps, start=None):
        step = self.step
        if not host_steps:
            return None
        uploaded = self._upload(0, host_steps[0][0], host_steps[0][1], after=start)
        for k, (inputs, v_img, outputs) in enumerate(host_steps):
            p = k % 2
            self.compute.wait_event(uploaded)
            if k + 1 < len(host_steps):
                nxt = host_steps[k + 1]
                uploaded = self._upload(k + 1, nxt[0], nxt[1])
            if self.out_free[p] is not None:
                self.compute.wait_event(self.out_free[p])
            for name in self.GRADS:
                setattr(step, name, self.dev_out[p][name])
            step.forward(*self.dev_in[p])
            step.backward(self.dev_vimg[p])
            done = torch.cuda.Event()
            done.record(self.compute)
            self.in_free[p] = done
            fin = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(self.down):
                self.down.wait_event(done)
                for name in self.GRADS:
                    outputs[name].copy_(self.dev_out[p][name], non_blocking=True)
                fin.record(self.down)
            self.out_free[p] = fin
        return self.out_free[(len(host_steps) - 1) % 2]

    def sync(self):
        torch.cuda.synchronize(self.step.dev)
