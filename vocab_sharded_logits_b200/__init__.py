"""Vocab-sliced logits and per-row sampler for one NVIDIA B200 (sm_100a).

A thin binding over the C ABI of ``libvsl.so`` (``include/vsl.h``): argument
marshalling only; every step of the path runs in the library's CUDA kernels.
PyTorch is used for device memory and streams.  There is no fallback: if the
library is missing, importing the binding raises.
"""
import ctypes
import os

import torch

__all__ = [
    "logits_local", "tile_stats", "tile_stats_shape", "sample", "sample_launches", "sample_plan", "make_row_params", "SampleResult", "lib", "status_string",
    "device_error", "VslError", "verify_drafts", "VerifyResult", "MAX_SPEC", "ROW_NONFINITE", "ROW_ALL_NEG_INF", "ROW_BAD_TEMPERATURE",
    "ROW_BAD_TOP_P", "ROW_BAD_TOP_K", "ROW_SCALE_OVERFLOW", "MAX_SLICES", "MAX_LOGPROBS",
]

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libvsl.so")

MAX_SLICES = 16
MAX_LOGPROBS = 20
MAX_SPEC = 64
ROW_NONFINITE = 1 << 0
ROW_ALL_NEG_INF = 1 << 1
ROW_BAD_TEMPERATURE = 1 << 2
ROW_BAD_TOP_P = 1 << 3
ROW_BAD_TOP_K = 1 << 4
ROW_SCALE_OVERFLOW = 1 << 5

_STATUS_NAMES = {0: "VSL_OK", 1: "VSL_ERR_INVALID_ARG", 2: "VSL_ERR_ALIGNMENT", 3: "VSL_ERR_UNSUPPORTED",
                 4: "VSL_ERR_WORKSPACE_TOO_SMALL", 5: "VSL_ERR_CUDA", 6: "VSL_ERR_DEVICE_TIMEOUT"}


class VslError(RuntimeError):
    """A libvsl call returned a status other than VSL_OK (``status`` is the code)."""

    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {_STATUS_NAMES.get(status, status)} ({status_string(status)})")


class _Extras(ctypes.Structure):
    _fields_ = [("kept_theta", ctypes.c_void_p), ("processed_logprob", ctypes.c_void_p),
                ("processed_topn_ids", ctypes.c_void_p), ("processed_topn_logprob", ctypes.c_void_p),
                ("tile_stats", ctypes.c_void_p)]


class _Plan(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in (
        "launches", "side_by_side", "stream_cluster", "stream_part", "stream_grid", "cluster", "part",
        "others_grid", "deferred_grid")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libvsl.so not built at {LIB_PATH}; run vocab_sharded_logits_b200/build.py")
    l = ctypes.CDLL(LIB_PATH)
    vp, i32, u32, u64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_size_t
    l.vsl_logits_local.restype = ctypes.c_int
    l.vsl_logits_local.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i32, i32, i32, vp]
    l.vsl_logits_local_ex.restype = ctypes.c_int
    l.vsl_logits_local_ex.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i32, i32, i32, vp, vp]
    l.vsl_tile_stats_floats.restype = sz
    l.vsl_tile_stats_floats.argtypes = [i32, i32, i32]
    l.vsl_tile_stats.restype = ctypes.c_int
    l.vsl_tile_stats.argtypes = [ctypes.POINTER(vp), i32, i32, i32, vp, vp]
    l.vsl_sample_workspace_bytes.restype = sz
    l.vsl_sample_workspace_bytes.argtypes = [i32, i32, i32, i32]
    l.vsl_sample_launches.restype = i32
    l.vsl_sample_launches.argtypes = [i32, i32, i32]
    l.vsl_sample_plan_for.restype = ctypes.c_int
    l.vsl_sample_plan_for.argtypes = [i32, i32, i32, i32, i32, ctypes.POINTER(_Plan)]
    l.vsl_sample.restype = ctypes.c_int
    l.vsl_sample.argtypes = [ctypes.POINTER(vp), i32, i32, i32, vp, u64, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    l.vsl_sample_ex.restype = ctypes.c_int
    l.vsl_sample_ex.argtypes = [ctypes.POINTER(vp), i32, i32, i32, vp, u64, i32, vp, vp, vp, vp, vp, vp, sz,
                                ctypes.POINTER(_Extras), vp]
    l.vsl_verify_drafts.restype = ctypes.c_int
    l.vsl_verify_drafts.argtypes = [vp, vp, vp, i32, i32, vp, vp, vp, vp]
    l.vsl_device_error.restype = ctypes.c_int
    l.vsl_device_error.argtypes = [ctypes.POINTER(u32)]
    l.vsl_status_string.restype = ctypes.c_char_p
    l.vsl_status_string.argtypes = [ctypes.c_int]
    l.vsl_version.restype = ctypes.c_char_p
    l.vsl_version.argtypes = []
    return l


lib = _load()


def status_string(status):
    return lib.vsl_status_string(int(status)).decode()


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _ptr_array(ts):
    arr = (ctypes.c_void_p * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = t.data_ptr()
    return arr


def _stream_handle(stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _check(status, where):
    if status != 0:
        raise VslError(status, where)


def _on_device(device):
    """The library launches on the current device: make the tensors' device current."""
    if device.type != "cuda":
        raise ValueError(f"libvsl needs CUDA tensors, got a tensor on {device}")
    return torch.cuda.device(device)


def tile_stats_shape(R, S, V_s):
    """Shape of the tile statistics of R rows of S slices of V_s logits: [R, S * B, 8],
    B = ceil(V_s / 128) (one record per block of 128 ids; ``include/vsl.h``)."""
    return (R, S * (-(-V_s // 128)), 8)


def _stats_tensor(stats, R, S, V_s, dev):
    shape = tile_stats_shape(R, S, V_s)
    if stats is True:
        return torch.empty(shape, dtype=torch.float32, device=dev)
    if stats.dtype != torch.float32 or tuple(stats.shape) != shape or not stats.is_contiguous() or stats.device != dev:
        raise ValueError(f"tile statistics must be a contiguous fp32 {list(shape)} tensor on {dev}")
    return stats


def tile_stats(logits_slices, out=None, stream=None):
    """Tile statistics of logits already in memory (fp32 [R, S * B, 8]; one read of the logits)."""
    R, V_s = logits_slices[0].shape
    S = len(logits_slices)
    dev = logits_slices[0].device
    for t in logits_slices:
        if t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != (R, V_s) or t.device != dev:
            raise ValueError("logits slices must be contiguous fp32 [R, V_s] on one device")
    out = _stats_tensor(True if out is None else out, R, S, V_s, dev)
    with _on_device(dev):
        status = lib.vsl_tile_stats(_ptr_array(logits_slices), R, S, V_s, _ptr(out), _stream_handle(stream, dev))
    _check(status, "vsl_tile_stats")
    return out


def logits_local(hidden, w_slices, out=None, stream=None, tile_stats=None):
    """Vocab-slice projection with no gather: ``out[s] = hidden @ w_slices[s].T`` in fp32.

    hidden: bf16 [R, H] CUDA tensor; w_slices: list of bf16 [V_s, H] CUDA tensors.
    Returns the list of fp32 [R, V_s] slices (``out`` if given).  With ``tile_stats``
    (True, or an fp32 [R, S * B, 8] tensor to fill) the projection also writes the
    tile statistics of its logits, and the call returns ``(slices, stats)``.
    """
    R, H = hidden.shape
    S = len(w_slices)
    V_s = w_slices[0].shape[0]
    if out is None:
        out = [torch.empty(R, V_s, dtype=torch.float32, device=hidden.device) for _ in range(S)]
    for t in [hidden, *w_slices, *out]:
        if not t.is_contiguous():
            raise ValueError("logits_local needs contiguous tensors")
    if hidden.dtype != torch.bfloat16 or any(w.dtype != torch.bfloat16 for w in w_slices):
        raise TypeError("hidden and weights must be bfloat16")
    for t in [*w_slices, *out]:
        if t.device != hidden.device:
            raise ValueError("logits_local: every tensor must be on the hidden states' device")
    stats = None if tile_stats is None or tile_stats is False else _stats_tensor(tile_stats, R, S, V_s, hidden.device)
    with _on_device(hidden.device):
        status = lib.vsl_logits_local_ex(_ptr(hidden), _ptr_array(w_slices), _ptr_array(out), R, H, S, V_s,
                                         _ptr(stats), _stream_handle(stream, hidden.device))
    _check(status, "vsl_logits_local")
    return out if stats is None else (out, stats)


def make_row_params(temperature, top_k, top_p, request_id, position, device):
    """Pack per-row parameters into the 20-byte ``vsl_row_params`` layout (int32 [R, 5])."""
    t = torch.as_tensor(temperature, dtype=torch.float32).reshape(-1)
    R = t.numel()
    k = torch.as_tensor(top_k, dtype=torch.int32).reshape(-1).expand(R)
    p = torch.as_tensor(top_p, dtype=torch.float32).reshape(-1).expand(R)
    req = torch.as_tensor(request_id, dtype=torch.int64).reshape(-1).expand(R)
    pos = torch.as_tensor(position, dtype=torch.int64).reshape(-1).expand(R)
    packed = torch.empty(R, 5, dtype=torch.int32)
    packed[:, 0] = t.view(torch.int32)
    packed[:, 1] = k
    packed[:, 2] = p.contiguous().view(torch.int32)
    packed[:, 3] = _u32_to_i32(req)
    packed[:, 4] = _u32_to_i32(pos)
    return packed.to(device)


def _u32_to_i32(x):
    x = x & 0xFFFFFFFF
    return torch.where(x >= 2 ** 31, x - 2 ** 32, x).to(torch.int32)


class SampleResult:
    """Outputs of ``sample``: token ids, their raw logprobs, top-n ids / logprobs, row
    flags, and (when asked for) the kept-set thresholds ``kept_theta`` [R, 2]."""

    def __init__(self, token_ids, token_logprob, topn_ids, topn_logprob, row_flags, kept_theta=None,
                 processed_logprob=None, processed_topn_ids=None, processed_topn_logprob=None):
        self.token_ids = token_ids
        self.token_logprob = token_logprob
        self.topn_ids = topn_ids
        self.topn_logprob = topn_logprob
        self.row_flags = row_flags
        self.kept_theta = kept_theta
        self.processed_logprob = processed_logprob
        self.processed_topn_ids = processed_topn_ids
        self.processed_topn_logprob = processed_topn_logprob


def sample(logits_slices, params, seed, n_logprobs, out=None, stream=None, kept_theta=False, processed=False,
           tile_stats=None):
    """Per-row temperature / top-k / top-p / Gumbel-max draw / top-n raw logprobs.

    logits_slices: list of fp32 [R, V_s] CUDA tensors (row r = concatenation over slices).
    params: int32 [R, 5] CUDA tensor from ``make_row_params``.
    kept_theta: also return each row's (theta_k, theta_p) on x = fl(l / T) (fp32 [R, 2]):
    the draw's kept set is every finite x >= max(theta_k, theta_p); -inf for a rule
    that is off, NaN for greedy and flagged rows.
    processed: also return the processed logprobs (log-probabilities of the distribution
    each token was drawn from: the token's [R], the top-n ids / values [R, n]); implies
    kept_theta.
    tile_stats: the tile statistics of exactly these logits (``logits_local(...,
    tile_stats=True)`` or ``tile_stats``): greedy and top-k rows then read only the
    quarters that can hold their candidates.
    """
    R, V_s = logits_slices[0].shape
    S = len(logits_slices)
    dev = logits_slices[0].device
    for t in logits_slices:
        if t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != (R, V_s) or t.device != dev:
            raise ValueError("logits slices must be contiguous fp32 [R, V_s] on one device")
    if params.dtype != torch.int32 or tuple(params.shape) != (R, 5) or not params.is_contiguous():
        raise ValueError("params must be a contiguous int32 [R, 5] tensor (make_row_params)")
    if out is None:
        n = max(n_logprobs, 1)
        out = SampleResult(torch.empty(R, dtype=torch.int32, device=dev),
                           torch.empty(R, dtype=torch.float32, device=dev),
                           torch.empty(R, n, dtype=torch.int32, device=dev)[:, :n_logprobs],
                           torch.empty(R, n, dtype=torch.float32, device=dev)[:, :n_logprobs],
                           torch.empty(R, dtype=torch.int32, device=dev))
    if params.device != dev:
        raise ValueError("params must be on the logits' device")
    kept_theta = kept_theta or processed
    if kept_theta and out.kept_theta is None:
        out.kept_theta = torch.empty(R, 2, dtype=torch.float32, device=dev)
    if processed and out.processed_logprob is None:
        n = max(n_logprobs, 1)
        out.processed_logprob = torch.empty(R, dtype=torch.float32, device=dev)
        out.processed_topn_ids = torch.empty(R, n, dtype=torch.int32, device=dev)[:, :n_logprobs]
        out.processed_topn_logprob = torch.empty(R, n, dtype=torch.float32, device=dev)[:, :n_logprobs]
    extras = None
    if tile_stats is not None:
        if not isinstance(tile_stats, torch.Tensor):
            raise TypeError("tile_stats must be the statistics tensor of these logits")
        tile_stats = _stats_tensor(tile_stats, R, S, V_s, dev)
        extras = _Extras()
        extras.tile_stats = tile_stats.data_ptr()
    if kept_theta:
        if out.kept_theta.dtype != torch.float32 or tuple(out.kept_theta.shape) != (R, 2) or \
                not out.kept_theta.is_contiguous():
            raise ValueError("kept_theta must be a contiguous fp32 [R, 2] tensor")
        extras = extras if extras is not None else _Extras()
        extras.kept_theta = out.kept_theta.data_ptr()
    if processed:
        extras.processed_logprob = out.processed_logprob.data_ptr()
        if n_logprobs > 0:
            extras.processed_topn_ids = out.processed_topn_ids.data_ptr()
            extras.processed_topn_logprob = out.processed_topn_logprob.data_ptr()
    ws_bytes = lib.vsl_sample_workspace_bytes(R, S, V_s, n_logprobs)
    with _on_device(dev):
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
        topn_ids = out.topn_ids if n_logprobs > 0 else None
        topn_lp = out.topn_logprob if n_logprobs > 0 else None
        status = lib.vsl_sample_ex(_ptr_array(logits_slices), R, S, V_s, _ptr(params),
                                   ctypes.c_uint64(seed & (2 ** 64 - 1)), n_logprobs, _ptr(out.token_ids),
                                   _ptr(out.token_logprob), _ptr(topn_ids), _ptr(topn_lp), _ptr(out.row_flags),
                                   _ptr(ws), ws_bytes, ctypes.byref(extras) if extras is not None else None,
                                   _stream_handle(stream, dev))
    _check(status, "vsl_sample")
    return out


class VerifyResult:
    """Outputs of ``verify_drafts``: accepted drafts per request, the emitted
    tokens [requests, spec + 1] and (when asked for) their logprobs."""

    def __init__(self, accepted, out_ids, out_logprob=None):
        self.accepted = accepted
        self.out_ids = out_ids
        self.out_logprob = out_logprob


def verify_drafts(token_ids, draft_ids, token_logprob=None, out=None, stream=None):
    """Speculative verification of deterministic drafts over ``sample``'s rows.

    token_ids: int32 [requests * (spec + 1)] CUDA tensor (``sample``'s tokens, rows of a
    request consecutive); draft_ids: int32 [requests, spec] CUDA tensor; token_logprob:
    optional fp32 [requests * (spec + 1)].  Draft j is accepted while the target's draw
    at position j equals it; a request emits its accepted drafts, then the target's
    token at the first rejected position (or the bonus token), then -1.
    """
    requests, spec = draft_ids.shape
    dev = token_ids.device
    if token_ids.dtype != torch.int32 or token_ids.numel() != requests * (spec + 1) or not token_ids.is_contiguous():
        raise ValueError("token_ids must be a contiguous int32 tensor of requests * (spec + 1) rows")
    if draft_ids.dtype != torch.int32 or not draft_ids.is_contiguous() or draft_ids.device != dev:
        raise ValueError("draft_ids must be a contiguous int32 [requests, spec] tensor on the tokens' device")
    if token_logprob is not None and (token_logprob.dtype != torch.float32 or not token_logprob.is_contiguous()
                                      or token_logprob.numel() != token_ids.numel() or token_logprob.device != dev):
        raise ValueError("token_logprob must be a contiguous fp32 tensor like token_ids")
    if out is None:
        out = VerifyResult(torch.empty(requests, dtype=torch.int32, device=dev),
                           torch.empty(requests, spec + 1, dtype=torch.int32, device=dev),
                           torch.empty(requests, spec + 1, device=dev) if token_logprob is not None else None)
    with _on_device(dev):
        status = lib.vsl_verify_drafts(_ptr(token_ids), _ptr(token_logprob), _ptr(draft_ids) if spec else None,
                                       requests, spec, _ptr(out.out_ids),
                                       _ptr(out.out_logprob) if token_logprob is not None else None,
                                       _ptr(out.accepted), _stream_handle(stream, dev))
    _check(status, "vsl_verify_drafts")
    return out


def sample_launches(R, S, V_s):
    """Kernels one ``sample`` call with these sizes launches on the current device."""
    n = lib.vsl_sample_launches(int(R), int(S), int(V_s))
    if n < 0:
        raise ValueError(f"vsl_sample_launches: sizes rejected (R={R}, S={S}, V_s={V_s})")
    return n


def sample_plan(R, S, V_s, sms, max_cluster):
    """The launches ``sample`` makes for these sizes on a device with ``sms`` SMs that
    schedules clusters of at most ``max_cluster`` CTAs, as a dict (host only)."""
    p = _Plan()
    _check(lib.vsl_sample_plan_for(int(R), int(S), int(V_s), int(sms), int(max_cluster), ctypes.byref(p)),
           "vsl_sample_plan_for")
    return {name: getattr(p, name) for name, _ in _Plan._fields_}


def device_error():
    """Reads and clears the kernels' error word (synchronises the device)."""
    code = ctypes.c_uint32(0)
    status = lib.vsl_device_error(ctypes.byref(code))
    return status, code.value
