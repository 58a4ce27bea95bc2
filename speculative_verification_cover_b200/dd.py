"""ctypes binding of libdd.so (include/dd.h), one Python function per C entry point.

Argument marshalling only: sizes are read off the tensors, pointers passed
as `data_ptr()`, the stream defaults to torch's current CUDA stream. Every
computation runs in libdd's CUDA kernels; there is no CPU fallback -- CPU
tensors, a missing library or a non-OK status raise.

With DD_CHECK_BOUNDS=1 in the environment (read when the library is first
loaded) the binding loads libdd_checked.so, the same library built with device
index checks (see dd_bounds_checked in include/dd.h).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, fields

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdd.so")
CHECKED_LIB_PATH = os.path.join(_HERE, "libdd_checked.so")

DD_OK, DD_ERR_INVALID_ARG, DD_ERR_UNSUPPORTED, DD_ERR_CUDA, DD_ERR_TIMEOUT, DD_ERR_BOUNDS = range(6)
DD_F32, DD_BF16 = 0, 1
POLICIES = {"trust": 0, "kl": 1, "conf": 2, "cover": 3, "coupled": 4, "kl_stochastic": 5}
DD_NONE, DD_KEEP, DD_REPLACE, DD_REMASK, DD_COMMIT = 0, 1, 2, 3, 4
DD_MASK_TOKEN = -1

# Every symbol include/dd.h declares.
EXPORTED = (
    "dd_dualview_attention", "dd_dualview_attention_ex", "dd_dualview_attention_ex2",
    "dd_dualview_attention_workspace_size", "dd_verify_logits",
    "dd_verify_logits_workspace_size", "dd_verify_logits_static",
    "dd_coupled_gumbel", "dd_select_seeds", "dd_select_seeds_ex", "dd_decide",
    "dd_status_string",
    "dd_get_device_error", "dd_set_spin_limit", "dd_selftest_bounded_wait",
    "dd_selftest_gumbel_screen", "dd_bounds_checked", "dd_selftest_bounds_check",
)


class DDError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")


class _RowStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "lse_t", "lse_d", "conf_t", "p_sample_t", "entropy_t", "kl_dt",
        "argmax_t", "argmax_d", "sample_t", "sample_d")]


class _DecideParams(ctypes.Structure):
    _fields_ = [("policy", ctypes.c_int), ("tau_kl", ctypes.c_float),
                ("tau_conf", ctypes.c_float), ("temperature", ctypes.c_float),
                ("tau_commit", ctypes.c_float), ("min_commit", ctypes.c_int),
                ("seed", ctypes.c_uint64), ("step", ctypes.c_uint64)]


_lib = None


def lib_path() -> str:
    """The library lib() loads: the checked build when DD_CHECK_BOUNDS is set to
    anything but 0 or the empty string, libdd.so otherwise."""
    return CHECKED_LIB_PATH if os.environ.get("DD_CHECK_BOUNDS", "0") not in ("", "0") else LIB_PATH


def lib():
    """Load the library (once). Raises ImportError if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m speculative_verification_cover_b200.build`")
    L = ctypes.CDLL(path)
    P, I, I64, U64, F, SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                             ctypes.c_float, ctypes.c_size_t)
    L.dd_dualview_attention.argtypes = [P] * 8 + [I] * 5 + [F, I, I] + [P] * 5 + [SZ, P]
    L.dd_dualview_attention.restype = I
    L.dd_dualview_attention_ex.argtypes = [P] * 8 + [I] * 5 + [F, I, I, I, F] + [P] * 5 + [SZ, P]
    L.dd_dualview_attention_ex.restype = I
    L.dd_dualview_attention_ex2.argtypes = [P] * 8 + [I] * 5 + [F, I, I, I, F] + [P] * 5 + [SZ, P, P]
    L.dd_dualview_attention_ex2.restype = I
    L.dd_dualview_attention_workspace_size.argtypes = [I] * 5
    L.dd_dualview_attention_workspace_size.restype = SZ
    L.dd_verify_logits.argtypes = [P, P, I, I, I, I, I64, I, F, U64, U64,
                                   ctypes.POINTER(_RowStats), P, SZ, P]
    L.dd_verify_logits.restype = I
    L.dd_verify_logits_static.argtypes = [P, P, I, I, I, I, I64, I, F, U64, U64,
                                          ctypes.POINTER(_RowStats), P]
    L.dd_verify_logits_static.restype = I
    L.dd_verify_logits_workspace_size.argtypes = [I, I, I, I]
    L.dd_verify_logits_workspace_size.restype = SZ
    L.dd_coupled_gumbel.argtypes = [U64, U64, I, I, I, I64, I, P, P]
    L.dd_coupled_gumbel.restype = I
    L.dd_select_seeds.argtypes = [P, I, I, P, P, P, I, I, I, P, P, P, P]
    L.dd_select_seeds.restype = I
    L.dd_select_seeds_ex.argtypes = [P, I, I, P, P, P, I, I, I, F, P, P, P, P, P]
    L.dd_select_seeds_ex.restype = I
    L.dd_decide.argtypes = [ctypes.POINTER(_DecideParams), P, P, P, ctypes.POINTER(_RowStats),
                            I, I, I, I, P, P, P, P]
    L.dd_decide.restype = I
    L.dd_status_string.argtypes = [I]
    L.dd_status_string.restype = ctypes.c_char_p
    L.dd_get_device_error.argtypes = [P]
    L.dd_get_device_error.restype = I
    L.dd_set_spin_limit.argtypes = [ctypes.c_uint32]
    L.dd_set_spin_limit.restype = ctypes.c_uint32
    L.dd_selftest_bounded_wait.argtypes = [ctypes.c_uint32, P]
    L.dd_selftest_bounded_wait.restype = I
    L.dd_selftest_gumbel_screen.argtypes = [P, P, P, P, I, ctypes.POINTER(F), P]
    L.dd_selftest_gumbel_screen.restype = I
    L.dd_bounds_checked.argtypes = []
    L.dd_bounds_checked.restype = I
    L.dd_selftest_bounds_check.argtypes = [I, I, ctypes.POINTER(I), P]
    L.dd_selftest_bounds_check.restype = I
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().dd_status_string(int(status)).decode()


def _check(fn, status):
    if status != DD_OK:
        raise DDError(fn, status)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("libdd takes device memory: tensor is on the CPU")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _dtype_code(t):
    if t.dtype == torch.float32:
        return DD_F32
    if t.dtype == torch.bfloat16:
        return DD_BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


@dataclass
class RowStats:
    """Per-row outputs of dd_verify_logits, each a [B, R] device tensor (or None)."""
    lse_t: torch.Tensor | None = None
    lse_d: torch.Tensor | None = None
    conf_t: torch.Tensor | None = None
    p_sample_t: torch.Tensor | None = None
    entropy_t: torch.Tensor | None = None
    kl_dt: torch.Tensor | None = None
    argmax_t: torch.Tensor | None = None
    argmax_d: torch.Tensor | None = None
    sample_t: torch.Tensor | None = None
    sample_d: torch.Tensor | None = None

    @classmethod
    def empty(cls, B, R, device="cuda"):
        f = dict(dtype=torch.float32, device=device)
        i = dict(dtype=torch.int32, device=device)
        return cls(*(torch.empty(B, R, **f) for _ in range(6)),
                   *(torch.empty(B, R, **i) for _ in range(4)))

    def _c(self):
        return _RowStats(*(_ptr(getattr(self, f.name)) for f in fields(self)))


def dd_dualview_attention_workspace_size(B, L, Hq, Hkv, d) -> int:
    return int(lib().dd_dualview_attention_workspace_size(B, L, Hq, Hkv, d))


def dd_dualview_attention(q, k_cur, v_cur, k_prev, v_prev, is_seed, is_masked, is_new,
                          out, lse, d_in=None, d_out=None, workspace=None, softmax_scale=0.0,
                          accumulate_stats=False, stream=None):
    """q [B,L,Hq,d]; k/v [B,L,Hkv,d]; masks [B,L] uint8; out like q; lse [B,Hq,L] fp32;
    d_in, d_out [B,L] fp32; workspace: uint8 device tensor of
    dd_dualview_attention_workspace_size(...) bytes."""
    B, L, Hq, d = q.shape
    Hkv = k_cur.shape[2]
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib().dd_dualview_attention(
        _ptr(q), _ptr(k_cur), _ptr(v_cur), _ptr(k_prev), _ptr(v_prev), _ptr(is_seed),
        _ptr(is_masked), _ptr(is_new), B, L, Hq, Hkv, d, float(softmax_scale), _dtype_code(q),
        int(bool(accumulate_stats)), _ptr(out), _ptr(lse), _ptr(d_in), _ptr(d_out),
        _ptr(workspace), nbytes, _stream(stream))
    _check("dd_dualview_attention", st)


def dd_dualview_attention_ex(q, k_cur, v_cur, k_prev, v_prev, is_seed, is_masked, is_new,
                             out, lse, d_in=None, d_out=None, workspace=None, q_begin=0,
                             accumulate_stats=False, stats_weight=1.0, softmax_scale=0.0,
                             stream=None, prep_done=None):
    """One layer of a multi-layer pass with a prefix cache: query rows from q_begin on,
    this layer's d_in / d_out weighted by stats_weight (see include/dd.h). prep_done: a
    torch.cuda.Event recorded right after the mask preparation (dd_dualview_attention_ex2)."""
    B, L, Hq, d = q.shape
    Hkv = k_cur.shape[2]
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    args = (_ptr(q), _ptr(k_cur), _ptr(v_cur), _ptr(k_prev), _ptr(v_prev), _ptr(is_seed),
            _ptr(is_masked), _ptr(is_new), B, L, Hq, Hkv, d, float(softmax_scale), _dtype_code(q),
            int(q_begin), int(bool(accumulate_stats)), float(stats_weight), _ptr(out), _ptr(lse),
            _ptr(d_in), _ptr(d_out), _ptr(workspace), nbytes)
    if prep_done is None:
        st = lib().dd_dualview_attention_ex(*args, _stream(stream))
        _check("dd_dualview_attention_ex", st)
    else:
        if not prep_done.cuda_event:
            raise ValueError("prep_done has no CUDA event yet: record it once first")
        st = lib().dd_dualview_attention_ex2(*args, ctypes.c_void_p(prep_done.cuda_event),
                                             _stream(stream))
        _check("dd_dualview_attention_ex2", st)


def dd_verify_logits_workspace_size(B, R, V, dtype) -> int:
    code = dtype if isinstance(dtype, int) else _dtype_code(torch.empty(0, dtype=dtype))
    return int(lib().dd_verify_logits_workspace_size(B, R, V, code))


def dd_verify_logits(logits_t, logits_d, out: RowStats, pos_offset=0, temperature=0.0, seed=0,
                     step=0, workspace=None, stream=None):
    """logits [B,R,V]; a view narrowed from a wider [B,R,ld] buffer is accepted
    (the row stride ld is read from the tensor). out: RowStats of [B,R] tensors.
    workspace: uint8 device tensor of dd_verify_logits_workspace_size(...) bytes
    (allocated here with torch when not given)."""
    B, R, V = logits_t.shape
    if workspace is None:
        workspace = torch.empty(dd_verify_logits_workspace_size(B, R, V, logits_t.dtype),
                                dtype=torch.uint8, device=logits_t.device)
    if logits_t.stride(2) != 1 or logits_t.stride(0) != R * logits_t.stride(1):
        raise ValueError("logits must be [B,R,V] with unit vocabulary stride and packed rows")
    if logits_d.shape != logits_t.shape or logits_d.stride() != logits_t.stride():
        raise ValueError("verifier and drafter logits must have the same shape and strides")
    if not (logits_t.is_cuda and logits_d.is_cuda):
        raise ValueError("libdd takes device memory: logits are on the CPU")
    ld = logits_t.stride(1)
    st = lib().dd_verify_logits(
        ctypes.c_void_p(logits_t.data_ptr()), ctypes.c_void_p(logits_d.data_ptr()),
        _dtype_code(logits_t), B, R, V, ld, int(pos_offset), float(temperature),
        int(seed) & (2**64 - 1), int(step) & (2**64 - 1), ctypes.byref(out._c()),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check("dd_verify_logits", st)


def dd_verify_logits_static(logits_t, logits_d, out: RowStats, pos_offset=0, temperature=0.0,
                            seed=0, step=0, stream=None):
    """dd_verify_logits without a workspace: for callers that cannot allocate device
    memory, the partial states live in a fixed array inside libdd (see include/dd.h for
    its size limit and for why concurrent calls must not overlap)."""
    B, R, V = logits_t.shape
    if logits_t.stride(2) != 1 or logits_t.stride(0) != R * logits_t.stride(1):
        raise ValueError("logits must be [B,R,V] with unit vocabulary stride and packed rows")
    if logits_d.shape != logits_t.shape or logits_d.stride() != logits_t.stride():
        raise ValueError("verifier and drafter logits must have the same shape and strides")
    if not (logits_t.is_cuda and logits_d.is_cuda):
        raise ValueError("libdd takes device memory: logits are on the CPU")
    st = lib().dd_verify_logits_static(
        ctypes.c_void_p(logits_t.data_ptr()), ctypes.c_void_p(logits_d.data_ptr()),
        _dtype_code(logits_t), B, R, V, logits_t.stride(1), int(pos_offset), float(temperature),
        int(seed) & (2**64 - 1), int(step) & (2**64 - 1), ctypes.byref(out._c()), _stream(stream))
    _check("dd_verify_logits_static", st)


def dd_coupled_gumbel(g, seed=0, step=0, pos_offset=0, stream=None):
    """Fill g [B,R,V] fp32 with the shared Gumbel noise of dd_verify_logits."""
    B, R, V = g.shape
    st = lib().dd_coupled_gumbel(int(seed) & (2**64 - 1), int(step) & (2**64 - 1), B, R, V,
                                 g.stride(1), int(pos_offset), _ptr(g), _stream(stream))
    _check("dd_coupled_gumbel", st)


def dd_select_seeds(entropy, pos_offset, d_in, d_out, eligible, seeds, is_seed=None, score=None,
                    stream=None):
    """entropy [B,R]; d_in, d_out [B,L] fp32; eligible [B,L] u8; seeds [B,k] int32 out."""
    B, L = d_in.shape
    R = entropy.shape[1] if entropy is not None else 0
    k = seeds.shape[1] if seeds is not None else 0
    st = lib().dd_select_seeds(_ptr(entropy), R, int(pos_offset), _ptr(d_in), _ptr(d_out),
                               _ptr(eligible), B, L, k, _ptr(seeds), _ptr(is_seed), _ptr(score),
                               _stream(stream))
    _check("dd_select_seeds", st)


def dd_select_seeds_ex(entropy, pos_offset, d_in, d_out, eligible, seeds, is_seed=None,
                       score=None, count=None, min_score=float("-inf"), stream=None):
    """dd_select_seeds with an adaptive size: only scores >= min_score compete;
    count [B] int32 (optional) receives the number chosen per sequence."""
    B, L = d_in.shape
    R = entropy.shape[1] if entropy is not None else 0
    k = seeds.shape[1] if seeds is not None else 0
    st = lib().dd_select_seeds_ex(_ptr(entropy), R, int(pos_offset), _ptr(d_in), _ptr(d_out),
                                  _ptr(eligible), B, L, k, float(min_score), _ptr(seeds),
                                  _ptr(is_seed), _ptr(score), _ptr(count), _stream(stream))
    _check("dd_select_seeds_ex", st)


def dd_decide(policy, tokens, is_seed, eligible, stats: RowStats, pos_offset, decision,
              new_tokens, accepted=None, tau_kl=0.5, tau_conf=0.9, temperature=0.0,
              tau_commit=0.0, min_commit=0, seed=0, step=0, stream=None):
    """tokens [B,L] int32; stats from dd_verify_logits ([B,R]); decision [B,L] u8,
    new_tokens [B,L] int32, accepted [B] u8 outputs. tau_commit > 0 turns on dynamic
    threshold decoding of masked positions; seed / step key the draws of the
    stochastic KL policy."""
    B, L = tokens.shape
    ref = stats.argmax_t if stats.argmax_t is not None else stats.sample_t
    R = ref.shape[1]
    p = _DecideParams(POLICIES[policy] if isinstance(policy, str) else int(policy),
                      float(tau_kl), float(tau_conf), float(temperature), float(tau_commit),
                      int(min_commit), int(seed) & (2**64 - 1), int(step) & (2**64 - 1))
    st = lib().dd_decide(ctypes.byref(p), _ptr(tokens), _ptr(is_seed), _ptr(eligible),
                         ctypes.byref(stats._c()), B, L, R, int(pos_offset), _ptr(decision),
                         _ptr(new_tokens), _ptr(accepted), _stream(stream))
    _check("dd_decide", st)


def dd_get_device_error(stream=None) -> int:
    """Synchronise the stream; return and clear the device error word."""
    return int(lib().dd_get_device_error(_stream(stream)))


def dd_set_spin_limit(limit: int) -> int:
    return int(lib().dd_set_spin_limit(int(limit)))


def dd_selftest_bounded_wait(spin_limit: int, stream=None):
    _check("dd_selftest_bounded_wait", lib().dd_selftest_bounded_wait(int(spin_limit),
                                                                      _stream(stream)))


def dd_selftest_gumbel_screen(g_req, stream=None):
    """The library's fp32 noise and screen j of every noise level (2^23 each), the
    screen limit of each requested level g_req (fp32 device tensor), and the
    constant above which the noise is skipped outright."""
    dev = g_req.device
    g = torch.empty(1 << 23, dtype=torch.float32, device=dev)
    j = torch.empty(1 << 23, dtype=torch.float32, device=dev)
    limit = torch.empty_like(g_req)
    gmax = ctypes.c_float(0.0)
    _check("dd_selftest_gumbel_screen", lib().dd_selftest_gumbel_screen(
        _ptr(g), _ptr(j), _ptr(g_req), _ptr(limit), g_req.numel(), ctypes.byref(gmax),
        _stream(stream)))
    return g, j, limit, float(gmax.value)


def dd_bounds_checked() -> bool:
    """True when the loaded library is the checked build."""
    return bool(lib().dd_bounds_checked())


def dd_selftest_bounds_check(n: int, index: int, stream=None) -> int:
    """One checked read of element `index` of a 64-int library array (element i
    holds 3*i + 1) limited to its first n: the value, or -1 when the check skipped
    the read (dd_get_device_error then returns DD_ERR_BOUNDS)."""
    v = ctypes.c_int(0)
    _check("dd_selftest_bounds_check",
           lib().dd_selftest_bounds_check(int(n), int(index), ctypes.byref(v), _stream(stream)))
    return int(v.value)
