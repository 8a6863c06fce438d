"""ctypes binding of libwan (the C ABI declared in include/wan.h).

Argument marshalling only: the raw entry points keep the C names
(``wan_block_forward`` and so on) and take integer device addresses; the
torch helpers below them pull ``data_ptr()`` and the current CUDA stream out
of tensors and raise ``WanError`` on a nonzero status. Every computation runs
inside the library. Loading fails loudly if ``libwan.so`` has not been built.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libwan.so")

WAN_OK, WAN_EINVAL, WAN_EALIGN, WAN_EUNSUPPORTED, WAN_ECUDA, WAN_ETIMEOUT, WAN_EBOUNDS = 0, -1, -2, -3, -4, -5, -6
WAN_F32, WAN_BF16, WAN_FP8, WAN_FP8_ATTN = 0, 1, 2, 3
WAN_NOALLOC_WORKSPACE_BYTES = 16 << 20
(WAN_WS_ACT, WAN_WS_QKV, WAN_WS_O, WAN_WS_QC, WAN_WS_KVC, WAN_WS_OC, WAN_WS_H, WAN_WS_MOD,
 WAN_WS_STATS, WAN_WS_A8, WAN_WS_ASCALE, WAN_WS_ATTN8) = range(12)
(WAN_K_GEMM_TC, WAN_K_GEMM_SIMT, WAN_K_ATTN_SELF, WAN_K_ATTN_CROSS, WAN_K_ATTN_SIMT, WAN_K_LAYERNORM,
 WAN_K_QKNORM_ROPE, WAN_K_EULER, WAN_K_MISC, WAN_K_ATTN_TC, WAN_K_MODEL, WAN_K_QUANT) = range(12)
WAN_K_COUNT = 12
KERNEL_CLASS_NAMES = ("gemm_tc", "gemm_simt", "attn_self", "attn_cross", "attn_simt", "layernorm",
                      "qknorm_rope", "euler_cfg", "misc", "attn_tc", "model", "quant")
STATUS_NAMES = {0: "WAN_OK", -1: "WAN_EINVAL", -2: "WAN_EALIGN", -3: "WAN_EUNSUPPORTED",
                -4: "WAN_ECUDA", -5: "WAN_ETIMEOUT", -6: "WAN_EBOUNDS"}


class WanError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


class wan_dims(ctypes.Structure):
    _fields_ = [("F", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("dim", ctypes.c_int), ("heads", ctypes.c_int), ("ffn_dim", ctypes.c_int),
                ("text_len", ctypes.c_int), ("eps", ctypes.c_float), ("dtype", ctypes.c_int),
                ("e0_per_token", ctypes.c_int)]


WEIGHT_FIELDS = ("modulation", "wq", "bq", "wk", "bk", "wv", "bv", "wo", "bo", "gq", "gk",
                 "g3", "b3", "cwq", "cbq", "cwk", "cbk", "cwv", "cbv", "cwo", "cbo",
                 "cgq", "cgk", "w1", "b1", "w2", "b2", "w_scales")
# the ten projection matrices, in the order of wan_block_weights.w_scales
FP8_MATRICES = ("wq", "wk", "wv", "wo", "cwq", "cwk", "cwv", "cwo", "w1", "w2")


class wan_block_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS]


class wan_model_dims(ctypes.Structure):
    _fields_ = [("C_in", ctypes.c_int), ("C_out", ctypes.c_int), ("F", ctypes.c_int),
                ("H", ctypes.c_int), ("W", ctypes.c_int), ("dim", ctypes.c_int),
                ("heads", ctypes.c_int), ("ffn_dim", ctypes.c_int), ("text_len", ctypes.c_int),
                ("text_dim", ctypes.c_int), ("freq_dim", ctypes.c_int), ("eps", ctypes.c_float),
                ("dtype", ctypes.c_int), ("t_per_token", ctypes.c_int)]


MODEL_WEIGHT_FIELDS = ("patch_w", "patch_b", "text_w1", "text_b1", "text_w2", "text_b2",
                       "time_w1", "time_b1", "time_w2", "time_b2", "proj_w", "proj_b",
                       "head_mod", "head_w", "head_b")


class wan_model_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in MODEL_WEIGHT_FIELDS]


_c_int, _vp, _sz = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t

_SIGS = {
    "wan_last_error": (ctypes.c_char_p, []),
    "wan_rope_freqs": (_c_int, [_c_int, _c_int, ctypes.c_double, _vp, _vp]),
    "wan_block_workspace_bytes": (_sz, [ctypes.POINTER(wan_dims), _c_int]),
    "wan_block_workspace_offset": (_sz, [ctypes.POINTER(wan_dims), _c_int, _c_int]),
    "wan_block_forward": (_c_int, [ctypes.POINTER(wan_dims), _c_int, _vp, _vp, _vp, _vp,
                                   ctypes.POINTER(wan_block_weights), _vp, _c_int, _vp, _sz, _vp]),
    "wan_block_forward_noalloc": (_c_int, [ctypes.POINTER(wan_dims), _c_int, _vp, _vp, _vp, _vp,
                                           ctypes.POINTER(wan_block_weights), _vp, _c_int, _vp]),
    "wan_block_sp_workspace_bytes": (_sz, [ctypes.POINTER(wan_dims), _c_int, _c_int]),
    "wan_block_sp_qkv": (_c_int, [ctypes.POINTER(wan_dims), _c_int, _c_int, _c_int, _vp, _vp,
                                  ctypes.POINTER(wan_block_weights), _vp, _c_int, _vp, _vp, _sz, _vp]),
    "wan_block_sp_finish": (_c_int, [ctypes.POINTER(wan_dims), _c_int, _c_int, _vp, _vp, _vp, _vp,
                                     ctypes.POINTER(wan_block_weights), _vp, _vp, _sz, _vp]),
    "wan_permute_chunks": (_c_int, [_vp, _vp, _c_int, ctypes.POINTER(ctypes.c_int),
                                    ctypes.POINTER(ctypes.c_int), _sz, _vp]),
    "wan_attention": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp,
                               _vp, ctypes.c_float, ctypes.POINTER(ctypes.c_int), _vp, _c_int, _vp]),
    "wan_euler_cfg_step": (_c_int, [_vp, _vp, _vp, _c_int, _sz, ctypes.c_float, ctypes.c_float,
                                    ctypes.c_float, _vp]),
    "wan_device_status": (_c_int, [_vp]),
    "wan_debug_bounds": (_c_int, []),
    "wan_profile_enable": (_c_int, [_c_int]),
    "wan_selftest_watchdog": (_c_int, [_vp]),
    "wan_profile_read": (_c_int, [_c_int, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]),
    "wan_model_workspace_bytes": (_sz, [ctypes.POINTER(wan_model_dims), _c_int]),
    "wan_quantize_fp8": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "wan_linear_fp8": (_c_int, [_c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "wan_attention_8bit_workspace_bytes": (_sz, [_c_int, _c_int, _c_int, _c_int]),
    "wan_unipc_coefficients": (_c_int, [ctypes.POINTER(ctypes.c_double), _c_int, _c_int, _c_int, _c_int,
                                        ctypes.POINTER(ctypes.c_double)]),
    "wan_unipc_step": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _sz, ctypes.c_float, ctypes.c_float,
                                ctypes.POINTER(ctypes.c_double), _vp]),
    "wan_attention_8bit": (_c_int, [_c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, ctypes.c_float,
                                    _vp, _sz, _vp]),
    "wan_model_forward": (_c_int, [ctypes.POINTER(wan_model_dims), _c_int, _vp, _vp, _vp, _vp,
                                   ctypes.POINTER(wan_model_weights),
                                   ctypes.POINTER(wan_block_weights), _c_int, _vp, _c_int, _vp,
                                   _vp, _sz, _vp]),
}

_lib = None


def load(path: str | None = None):
    """Load libwan.so (raises if it is missing: there is no fallback). The
    environment variable WAN_LIBRARY may name another build of the library
    (the debug build, ``build_lib.build(debug=True)``)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or os.environ.get("WAN_LIBRARY") or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"libwan.so not built at {path}; run "
                           "`python -m video_diffusion_transformer_fwd_b200.build_lib`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def wan_last_error() -> bytes:
    return load().wan_last_error()


def last_error() -> str:
    return wan_last_error().decode()


def check(rc: int):
    if rc != WAN_OK:
        raise WanError(rc, last_error())


# ---------------------------------------------------------------- raw C entry points
def wan_rope_freqs(head_dim, max_pos, theta, table, stream):
    return load().wan_rope_freqs(head_dim, max_pos, theta, table, stream)


def wan_block_workspace_bytes(dims, B):
    return load().wan_block_workspace_bytes(ctypes.byref(dims), B)


def wan_block_workspace_offset(dims, B, which):
    return load().wan_block_workspace_offset(ctypes.byref(dims), B, which)


def wan_block_forward(dims, B, x, ctx, ctx_lens, e0, weights, rope, rope_max_pos, workspace,
                      ws_bytes, stream):
    return load().wan_block_forward(ctypes.byref(dims), B, x, ctx, ctx_lens, e0,
                                    ctypes.byref(weights), rope, rope_max_pos, workspace,
                                    ws_bytes, stream)


def wan_block_forward_noalloc(dims, B, x, ctx, ctx_lens, e0, weights, rope, rope_max_pos, stream):
    return load().wan_block_forward_noalloc(ctypes.byref(dims), B, x, ctx, ctx_lens, e0,
                                            ctypes.byref(weights), rope, rope_max_pos, stream)


def wan_block_sp_workspace_bytes(dims, B, rows):
    return load().wan_block_sp_workspace_bytes(ctypes.byref(dims), B, rows)


def wan_block_sp_qkv(dims, B, rows, tok0, x, e0, weights, rope, rope_max_pos, qkv, workspace, ws_bytes,
                     stream):
    return load().wan_block_sp_qkv(ctypes.byref(dims), B, rows, tok0, x, e0, ctypes.byref(weights), rope,
                                   rope_max_pos, qkv, workspace, ws_bytes, stream)


def wan_block_sp_finish(dims, B, rows, x, ctx, ctx_lens, e0, weights, o, workspace, ws_bytes, stream):
    return load().wan_block_sp_finish(ctypes.byref(dims), B, rows, x, ctx, ctx_lens, e0, ctypes.byref(weights),
                                      o, workspace, ws_bytes, stream)


def wan_permute_chunks(src, dst, ndim, dims, perm, chunk_bytes, stream):
    d = (ctypes.c_int * max(ndim, 1))(*dims)
    p = (ctypes.c_int * max(ndim, 1))(*perm)
    return load().wan_permute_chunks(src, dst, ndim, d, p, chunk_bytes, stream)


def wan_attention(B, heads, Lq, Lk, head_dim, dtype, q, k, v, o, k_lens, scale, grid, rope,
                  rope_max_pos, stream):
    g = None if grid is None else (ctypes.c_int * 3)(*grid)
    return load().wan_attention(B, heads, Lq, Lk, head_dim, dtype, q, k, v, o, k_lens, scale,
                                g, rope, rope_max_pos, stream)


def wan_euler_cfg_step(x, v_cond, v_uncond, v_dtype, n, guide_scale, sigma, sigma_next, stream):
    return load().wan_euler_cfg_step(x, v_cond, v_uncond, v_dtype, n, guide_scale, sigma,
                                     sigma_next, stream)


def wan_model_workspace_bytes(dims, B):
    return load().wan_model_workspace_bytes(ctypes.byref(dims), B)


def wan_model_forward(dims, B, latent, t, text, ctx_lens, weights, blocks, num_blocks, rope,
                      rope_max_pos, out, workspace, ws_bytes, stream):
    return load().wan_model_forward(ctypes.byref(dims), B, latent, t, text, ctx_lens,
                                    ctypes.byref(weights), blocks, num_blocks, rope, rope_max_pos,
                                    out, workspace, ws_bytes, stream)


def wan_quantize_fp8(src, src_dtype, rows, cols, per_row, q, scale, stream):
    return load().wan_quantize_fp8(src, src_dtype, rows, cols, per_row, q, scale, stream)


def wan_linear_fp8(M, N, K, a, a_scale, w, w_scale, bias, out, stream):
    return load().wan_linear_fp8(M, N, K, a, a_scale, w, w_scale, bias, out, stream)


def wan_attention_8bit_workspace_bytes(B, heads, Lq, Lk):
    return load().wan_attention_8bit_workspace_bytes(B, heads, Lq, Lk)


def wan_attention_8bit(B, heads, Lq, Lk, q, k, v, o, k_lens, scale, workspace, ws_bytes, stream):
    return load().wan_attention_8bit(B, heads, Lq, Lk, q, k, v, o, k_lens, scale, workspace, ws_bytes,
                                     stream)


def wan_unipc_coefficients(sigmas, num_sigmas, step, order, lower_order_final, coef):
    return load().wan_unipc_coefficients(sigmas, num_sigmas, step, order, lower_order_final, coef)


def wan_unipc_step(x, last, m_out, m_prev1, m_prev2, v_cond, v_uncond, v_dtype, n, guide_scale, sigma, coef,
                   stream):
    return load().wan_unipc_step(x, last, m_out, m_prev1, m_prev2, v_cond, v_uncond, v_dtype, n, guide_scale,
                                 sigma, coef, stream)


def wan_debug_bounds():
    return load().wan_debug_bounds()


def wan_device_status(stream):
    return load().wan_device_status(stream)


def wan_selftest_watchdog(stream):
    return load().wan_selftest_watchdog(stream)


def wan_profile_enable(on):
    return load().wan_profile_enable(on)


def wan_profile_read(kernel_class, launches, total_ms):
    return load().wan_profile_read(kernel_class, launches, total_ms)


def profile_read():
    """{class name: (launches, total device ms)} of the current record."""
    out = {}
    for c in range(WAN_K_COUNT):
        n = ctypes.c_int(0)
        ms = ctypes.c_double(0.0)
        check(wan_profile_read(c, ctypes.byref(n), ctypes.byref(ms)))
        out[KERNEL_CLASS_NAMES[c]] = (n.value, ms.value)
    return out


# ---------------------------------------------------------------- torch helpers
def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return WAN_BF16
    if t.dtype == torch.float32:
        return WAN_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


DTYPE_CODES = {"bf16": WAN_BF16, "f32": WAN_F32, "fp8": WAN_FP8, "fp8attn": WAN_FP8_ATTN}


def make_dims(F, H, W, dim, heads, ffn_dim, text_len, eps=1e-6, dtype="bf16", e0_per_token=False) -> wan_dims:
    code = DTYPE_CODES[dtype] if isinstance(dtype, str) else int(dtype)
    return wan_dims(F, H, W, dim, heads, ffn_dim, text_len, eps, code, 1 if e0_per_token else 0)


def dims_of(cfg) -> wan_dims:
    return make_dims(cfg.F, cfg.H, cfg.W, cfg.dim, cfg.heads, cfg.ffn_dim, cfg.text_len,
                     cfg.eps, cfg.dtype)


def make_weights(w: dict) -> wan_block_weights:
    for n in WEIGHT_FIELDS:
        if w.get(n) is not None and not w[n].is_contiguous():
            raise ValueError(f"weight {n} must be contiguous")
    return wan_block_weights(*[_ptr(w.get(n)) for n in WEIGHT_FIELDS])


def quantize_fp8(t, per_row=True, stream=None):
    """e4m3 codes (uint8, same shape) and float32 scales ([rows] or [1]) of a
    float32 / bf16 tensor; rows are the last axis."""
    torch = _torch()
    cols = t.shape[-1] if t.dim() else 1
    rows = t.numel() // cols if cols else 0
    q = torch.empty(t.shape, dtype=torch.uint8, device=t.device)
    sc = torch.empty((rows if per_row else 1,), dtype=torch.float32, device=t.device)
    check(wan_quantize_fp8(t.data_ptr(), dtype_code(t), rows, cols, 1 if per_row else 0,
                           q.data_ptr(), sc.data_ptr(), _stream(stream)))
    return q, sc


def linear_fp8(a, a_scale, w, w_scale, bias=None, out=None, stream=None):
    """out = (a w^T) a_scale[m] w_scale + bias, float32 [M, N]."""
    torch = _torch()
    M, K = a.shape
    N = w.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=a.device)
    check(wan_linear_fp8(M, N, K, a.data_ptr(), a_scale.data_ptr(), w.data_ptr(), w_scale.data_ptr(),
                         _ptr(bias), out.data_ptr(), _stream(stream)))
    return out


def quantize_block_weights(w: dict, stream=None) -> dict:
    """An FP8 copy of a bf16 block weight dict: the ten projection matrices
    become e4m3 codes and ``w_scales`` holds their ten per-tensor scales."""
    torch = _torch()
    out = dict(w)
    scales = torch.empty(10, dtype=torch.float32, device=w["wq"].device)
    for i, n in enumerate(FP8_MATRICES):
        q, sc = quantize_fp8(w[n], per_row=False, stream=stream)
        out[n] = q
        scales[i:i + 1].copy_(sc)
    out["w_scales"] = scales
    return out


def rope_freqs(head_dim, max_pos=1024, theta=1e4, device="cuda", stream=None):
    torch = _torch()
    t = torch.empty((max_pos, head_dim // 2, 2), dtype=torch.float32, device=device)
    check(wan_rope_freqs(head_dim, max_pos, theta, t.data_ptr(), _stream(stream)))
    return t


def workspace_bytes(dims: wan_dims, B: int) -> int:
    n = wan_block_workspace_bytes(dims, B)
    if n == 0 and B > 0:
        raise WanError(WAN_EINVAL, last_error())
    return n


def alloc_workspace(dims: wan_dims, B: int, device="cuda"):
    torch = _torch()
    n = wan_block_workspace_bytes(dims, B)
    if n == 0:
        raise WanError(WAN_EINVAL, last_error())
    return torch.empty(n, dtype=torch.uint8, device=device)


def workspace_view(ws, dims: wan_dims, B: int, which: int, shape, dtype):
    """A tensor view of one workspace buffer (see WAN_WS_* in include/wan.h)."""
    torch = _torch()
    off = wan_block_workspace_offset(dims, B, which)
    n = 1
    for s in shape:
        n *= s
    es = torch.empty((), dtype=dtype).element_size()
    return ws[off:off + n * es].view(dtype).view(*shape)


def block_forward(dims: wan_dims, x, ctx, e0, weights, rope, workspace, ctx_lens=None,
                  stream=None, cweights=None):
    """One block in place on x ([B, L, dim] float32). ``weights`` is a dict of
    device tensors (see WEIGHT_FIELDS) or a prebuilt wan_block_weights."""
    B = x.shape[0]
    cw = weights if isinstance(weights, wan_block_weights) else make_weights(weights)
    check(wan_block_forward(dims, B, x.data_ptr(), _ptr(ctx), _ptr(ctx_lens), e0.data_ptr(), cw,
                            rope.data_ptr(), rope.shape[0], workspace.data_ptr(),
                            workspace.numel() * workspace.element_size(), _stream(stream)))
    return x


def attention(q, k, v, k_lens=None, scale=0.0, grid=None, rope=None, out=None, stream=None):
    """q [B, Lq, n, d], k/v [B, Lk, n, d] (bf16 or f32). With ``grid`` the
    3D RoPE is applied to q and k in place first."""
    torch = _torch()
    B, Lq, n, d = q.shape
    Lk = k.shape[1]
    o = torch.empty_like(q) if out is None else out
    check(wan_attention(B, n, Lq, Lk, d, dtype_code(q), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                        o.data_ptr(), _ptr(k_lens), scale, grid, _ptr(rope),
                        0 if rope is None else rope.shape[0], _stream(stream)))
    return o


def attention_8bit(q, k, v, k_lens=None, scale=0.0, out=None, workspace=None, stream=None):
    """8-bit attention: q [B, Lq, n, 128], k / v [B, Lk, n, 128] bf16."""
    torch = _torch()
    B, Lq, n, d = q.shape
    Lk = k.shape[1]
    o = torch.empty_like(q) if out is None else out
    if workspace is None:
        workspace = torch.empty(max(wan_attention_8bit_workspace_bytes(B, n, Lq, Lk), 1), dtype=torch.uint8,
                                device=q.device)
    check(wan_attention_8bit(B, n, Lq, Lk, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), _ptr(k_lens),
                             scale, workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return o


def euler_cfg_step(x, v_cond, v_uncond, guide_scale, sigma, sigma_next, stream=None):
    check(wan_euler_cfg_step(x.data_ptr(), v_cond.data_ptr(), _ptr(v_uncond), dtype_code(v_cond),
                             x.numel(), guide_scale, sigma, sigma_next, _stream(stream)))
    return x


def device_status(stream=None) -> int:
    return wan_device_status(_stream(stream))


def make_model_dims(C_in, C_out, F, H, W, dim, heads, ffn_dim, text_len, text_dim, freq_dim=256,
                    eps=1e-6, dtype="bf16", t_per_token=False) -> wan_model_dims:
    code = DTYPE_CODES[dtype] if isinstance(dtype, str) else int(dtype)
    return wan_model_dims(C_in, C_out, F, H, W, dim, heads, ffn_dim, text_len, text_dim, freq_dim,
                          eps, code, 1 if t_per_token else 0)


def make_model_weights(w: dict) -> wan_model_weights:
    for n in MODEL_WEIGHT_FIELDS:
        if w.get(n) is not None and not w[n].is_contiguous():
            raise ValueError(f"weight {n} must be contiguous")
    return wan_model_weights(*[_ptr(w.get(n)) for n in MODEL_WEIGHT_FIELDS])


def make_block_array(blocks) -> ctypes.Array:
    """A C array of wan_block_weights from a list of weight dicts (or structs)."""
    arr = (wan_block_weights * len(blocks))()
    for i, b in enumerate(blocks):
        arr[i] = b if isinstance(b, wan_block_weights) else make_weights(b)
    return arr


def alloc_model_workspace(dims: wan_model_dims, B: int, device="cuda"):
    torch = _torch()
    n = wan_model_workspace_bytes(dims, B)
    if n == 0:
        raise WanError(WAN_EINVAL, last_error())
    return torch.empty(n, dtype=torch.uint8, device=device)


def model_forward(dims: wan_model_dims, latent, t, text, weights, blocks, rope, workspace,
                  ctx_lens=None, out=None, stream=None):
    """Velocity of the whole model: latent [B, C_in, F, H, W] float32, t [B]
    (or [B, L] with dims.t_per_token) float32 timesteps (device), text [B, text_len, text_dim] in the compute
    dtype. ``blocks`` is a list of block weight dicts or a make_block_array()
    result. Returns out [B, C_out, F, H, W] float32."""
    torch = _torch()
    B = latent.shape[0]
    if out is None:
        out = torch.empty((B, dims.C_out, dims.F, dims.H, dims.W), dtype=torch.float32,
                          device=latent.device)
    mw = weights if isinstance(weights, wan_model_weights) else make_model_weights(weights)
    arr = blocks if isinstance(blocks, ctypes.Array) else make_block_array(blocks)
    check(wan_model_forward(dims, B, latent.data_ptr(), t.data_ptr(), _ptr(text), _ptr(ctx_lens),
                            mw, arr, len(arr), rope.data_ptr(), rope.shape[0],
                            out.data_ptr(), workspace.data_ptr(),
                            workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


class UniPCSampler:
    """State of the UniPC sampler over one latent (see wan_unipc_step): the
    schedule, the step index, the corrected previous sample and a ring of
    three data predictions. ``x`` (float32, device) is updated in place."""

    def __init__(self, x, sigmas, order=2, lower_order_final=True):
        torch = _torch()
        self.x = x
        self.sigmas = [float(s) for s in sigmas]
        self.n = len(self.sigmas) - 1
        self.order, self.lof = order, lower_order_final
        self.i = 0
        self.last = torch.empty_like(x)
        self.ring = [torch.empty_like(x) for _ in range(3)]
        self._sig = (ctypes.c_double * len(self.sigmas))(*self.sigmas)
        self._coef = (ctypes.c_double * 8)()

    @property
    def sigma(self) -> float:
        return self.sigmas[self.i]

    def coefficients(self, step=None):
        check(wan_unipc_coefficients(self._sig, len(self.sigmas), self.i if step is None else step, self.order,
                                     1 if self.lof else 0, self._coef))
        return list(self._coef)

    def step(self, v_cond, v_uncond=None, guide_scale=1.0, stream=None):
        if self.i >= self.n:
            raise RuntimeError("UniPC schedule finished")
        self.coefficients()
        i = self.i
        m_out = self.ring[i % 3]
        m1 = self.ring[(i - 1) % 3] if i >= 1 else None
        m2 = self.ring[(i - 2) % 3] if i >= 2 else None
        check(wan_unipc_step(self.x.data_ptr(), self.last.data_ptr(), m_out.data_ptr(), _ptr(m1), _ptr(m2),
                             v_cond.data_ptr(), _ptr(v_uncond), dtype_code(v_cond), self.x.numel(), guide_scale,
                             self.sigmas[i], self._coef, _stream(stream)))
        self.i += 1
        return self.x
