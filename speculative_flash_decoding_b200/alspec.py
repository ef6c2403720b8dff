"""ctypes binding of libalspec.so (the C ABI in include/alspec.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of libalspec.so.  There is no CPU fallback -- if the library is
missing or cannot be loaded, importing this module raises.

The functions named ``alspec_*`` mirror the C entry points one to one and
take plain integers (device pointers, stream/event handles) and sizes.
``Decoder`` is a convenience layer that takes torch tensors, owns a
workspace and raises ``AlspecError`` on a non-OK status.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
# ALSPEC_LIBRARY=debug loads the bounds-checked build of the same sources
# (libalspec_debug.so); the default is libalspec.so.
_LIBRARIES = {"": "libalspec.so", "default": "libalspec.so", "debug": "libalspec_debug.so"}
if os.environ.get("ALSPEC_LIBRARY", "") not in _LIBRARIES:
    raise ImportError("ALSPEC_LIBRARY must be unset, 'default' or 'debug', not "
                      f"{os.environ['ALSPEC_LIBRARY']!r}")
_LIB_NAME = _LIBRARIES[os.environ.get("ALSPEC_LIBRARY", "")]
LIB_PATH = os.path.join(_PKG, _LIB_NAME)

ALSPEC_OK = 0
ALSPEC_ERR_INVALID_ARG = 1
ALSPEC_ERR_UNSUPPORTED = 2
ALSPEC_ERR_WORKSPACE = 3
ALSPEC_ERR_CUDA = 4
ALSPEC_ERR_TIMEOUT = 5
ALSPEC_ERR_DEVICE_DATA = 6

ALSPEC_F32 = 0
ALSPEC_BF16 = 1

ALSPEC_PROF_EVENTS = 5

ALSPEC_DEVERR_SEQ_LEN = 0x1
ALSPEC_DEVERR_TIMEOUT = 0x2
ALSPEC_DEVERR_BOUNDS = 0x4   # bounds-checked debug build only

# Every symbol the header declares, with (restype, argtypes).
_vp, _i, _f, _sz, _u32p = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t,
                          ctypes.POINTER(ctypes.c_uint32))


ALSPEC_ENGINE_AUTO = 0
ALSPEC_ENGINE_CUDA_CORES = 1
ALSPEC_ENGINE_TENSOR_CORES = 2

ALSPEC_SCHEDULE_AUTO = 0
ALSPEC_SCHEDULE_STREAMS = 1
ALSPEC_SCHEDULE_FUSED = 2
ALSPEC_SCHEDULE_SINK_FIRST = 3


class alspec_desc(ctypes.Structure):
    _fields_ = [("batch", _i), ("n_q_heads", _i), ("n_kv_heads", _i), ("head_dim", _i),
                ("max_seq_len", _i), ("dtype", _i), ("split_tokens", _i), ("timeout_ms", _i),
                ("engine", _i), ("schedule", _i)]


_descp = ctypes.POINTER(alspec_desc)

SIGNATURES = {
    "alspec_workspace_size": (_sz, [_descp, _i, _i]),
    "alspec_workspace_init": (_i, [_vp, _sz, _vp]),
    "alspec_decode": (_i, [_descp, _vp, _vp, _vp, _vp, _i, _i, _f, _vp, _vp, _vp, _vp, _vp, _sz,
                           _vp, _vp, ctypes.POINTER(_vp)]),
    "alspec_query_plan": (_i, [_descp, _i, _i, ctypes.POINTER(_i), _i]),
    "alspec_get_device_error": (_i, [_vp, _sz, _vp, _u32p]),
    "alspec_query_chunks": (_i, [_descp, _i, _i, _u32p, _i, ctypes.POINTER(_i),
                                 ctypes.POINTER(_i)]),
    "alspec_graph_begin": (_i, [_vp]),
    "alspec_graph_end": (_i, [_vp, ctypes.POINTER(_vp)]),
    "alspec_graph_launch": (_i, [_vp, _vp]),
    "alspec_graph_destroy": (_i, [_vp]),
    "alspec_shutdown": (_i, []),
    "alspec_status_string": (ctypes.c_char_p, [_i]),
    "alspec_version": (_i, []),
    "alspec_last_cuda_error": (_i, []),
    "alspec_decode_noalloc": (_i, [_descp, _vp, _vp, _vp, _vp, _i, _i, _f, _vp, _vp, _vp, _vp,
                                   _vp]),
    "alspec_noalloc_device_error": (_i, [_vp, _u32p]),
    "alspec_decode_traced": (_i, [_descp, _vp, _vp, _vp, _vp, _i, _i, _f, _vp, _vp, _vp, _vp,
                                  _vp, _sz, _vp, _vp]),
    "alspec_oproj": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp]),
    "alspec_test_wait_timeout": (_i, [_vp, _sz, _i, _vp]),
    "alspec_decode_oproj": (_i, [_descp, _vp, _vp, _vp, _vp, _i, _i, _f, _vp, _i, _vp, _vp,
                                 _vp, _vp, _vp, _i, _vp, _sz, _vp, _vp]),
}

ALSPEC_NOALLOC_SCRATCH_BYTES = 8 << 20


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{_LIB_NAME} not found at {LIB_PATH}; build it with "
            "`python speculative_flash_decoding_b200/build.py` (there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


class AlspecError(RuntimeError):
    def __init__(self, status: int, where: str):
        extra = ""
        if status == ALSPEC_ERR_CUDA:
            extra = f", cudaError {alspec_last_cuda_error()}"
        super().__init__(f"{where}: {alspec_status_string(status)} (status {status}{extra})")
        self.status = status


# ------------------------------------------------------------ C entry points

def alspec_workspace_size(desc: alspec_desc, n_sink: int, window: int) -> int:
    return int(_lib.alspec_workspace_size(ctypes.byref(desc), n_sink, window))


def alspec_workspace_init(workspace: int, workspace_bytes: int, stream: int) -> int:
    return int(_lib.alspec_workspace_init(workspace, workspace_bytes, stream))


def alspec_decode(desc: alspec_desc, q: int, k_cache: int, v_cache: int, seq_lens: int,
                  n_sink: int, window: int, lam: float, out_spec: int, out_exact: int,
                  rel_l2: int, commit: int, workspace: int, workspace_bytes: int,
                  stream: int, spec_event: int = 0, prof_events=None) -> int:
    """prof_events: None or a sequence of ALSPEC_PROF_EVENTS event handles."""
    prof = None
    if prof_events is not None:
        prof = (ctypes.c_void_p * ALSPEC_PROF_EVENTS)(*[e or None for e in prof_events])
    return int(_lib.alspec_decode(ctypes.byref(desc), q, k_cache, v_cache, seq_lens, n_sink,
                                  window, lam, out_spec, out_exact, rel_l2, commit, workspace,
                                  workspace_bytes, stream, spec_event or None, prof))


def alspec_decode_traced(desc: alspec_desc, q: int, k_cache: int, v_cache: int, seq_lens: int,
                         n_sink: int, window: int, lam: float, out_spec: int, out_exact: int,
                         rel_l2: int, commit: int, workspace: int, workspace_bytes: int,
                         stream: int, trace_ns: int) -> int:
    """trace_ns: device address of 2 zeroed uint64 words; the kernels leave
    the global-timer ns of O_spec's and O_exact's publication there."""
    return int(_lib.alspec_decode_traced(ctypes.byref(desc), q, k_cache, v_cache, seq_lens,
                                         n_sink, window, lam, out_spec, out_exact, rel_l2,
                                         commit, workspace, workspace_bytes, stream,
                                         trace_ns or None))


def alspec_oproj(x: int, w: int, y: int, skip: int, batch: int, k: int, n: int,
                 stream: int, err: int = 0) -> int:
    """y[b, j] = sum_i x[b, i] * w[j, i]; rows with skip[b] != 0 untouched;
    err: device address of a uint32 error word, or 0."""
    return int(_lib.alspec_oproj(x, w, y, skip or None, batch, k, n, err or None, stream))


ALSPEC_GATE_KERNEL, ALSPEC_GATE_GRAPH_CONDITIONAL = 0, 1
GATES = {"kernel": ALSPEC_GATE_KERNEL, "graph_conditional": ALSPEC_GATE_GRAPH_CONDITIONAL}


def alspec_decode_oproj(desc: alspec_desc, q: int, k_cache: int, v_cache: int, seq_lens: int,
                        n_sink: int, window: int, lam: float, w_o: int, hidden: int,
                        out_spec: int, out_exact: int, rel_l2: int, commit: int, y: int,
                        gate: int, workspace: int, workspace_bytes: int, stream: int,
                        trace_ns: int = 0) -> int:
    """Decode plus the speculative output projection y = o_proj(O_spec or O_exact)."""
    return int(_lib.alspec_decode_oproj(ctypes.byref(desc), q, k_cache, v_cache, seq_lens,
                                        n_sink, window, lam, w_o, hidden, out_spec, out_exact,
                                        rel_l2, commit, y, gate, workspace, workspace_bytes,
                                        stream, trace_ns or None))


def alspec_test_wait_timeout(workspace: int, workspace_bytes: int, timeout_ms: int,
                             stream: int) -> int:
    """Test hook: a kernel whose waits can never complete must give up."""
    return int(_lib.alspec_test_wait_timeout(workspace, workspace_bytes, timeout_ms, stream))


def alspec_decode_noalloc(desc: alspec_desc, q: int, k_cache: int, v_cache: int, seq_lens: int,
                          n_sink: int, window: int, lam: float, out_spec: int, out_exact: int,
                          rel_l2: int, commit: int, stream: int) -> int:
    """alspec_decode without a workspace: for callers that cannot allocate
    device memory.  Uses the library's fixed 8 MiB device scratch array
    (shared by all calls on a device -- calls must not overlap on the GPU)."""
    return int(_lib.alspec_decode_noalloc(ctypes.byref(desc), q, k_cache, v_cache, seq_lens,
                                          n_sink, window, lam, out_spec, out_exact, rel_l2,
                                          commit, stream))


def alspec_noalloc_device_error(stream: int):
    """(status, error word) of alspec_decode_noalloc's scratch on the current
    device (read and cleared; synchronizes the stream)."""
    err = ctypes.c_uint32(0)
    st = int(_lib.alspec_noalloc_device_error(stream, ctypes.byref(err)))
    return st, int(err.value)


def alspec_query_plan(desc: alspec_desc, n_sink: int, window: int):
    info = (ctypes.c_int * 12)()
    st = int(_lib.alspec_query_plan(ctypes.byref(desc), n_sink, window, info, 12))
    keys = ("c1", "n1", "c2", "n2", "grid2", "threads", "smem", "stages", "engine", "schedule",
            "merge_c", "grid1")
    return st, dict(zip(keys, list(info)))


def alspec_query_chunks(desc: alspec_desc, n_sink: int, window: int):
    """(status, fq list of n2 + 1 fractions in 1/2^24, tile rows)."""
    cap = 257
    fq = (ctypes.c_uint32 * cap)()
    n2, tile = ctypes.c_int(0), ctypes.c_int(0)
    st = int(_lib.alspec_query_chunks(ctypes.byref(desc), n_sink, window, fq, cap,
                                      ctypes.byref(n2), ctypes.byref(tile)))
    return st, list(fq)[: n2.value + 1], tile.value


def alspec_get_device_error(workspace: int, workspace_bytes: int, stream: int):
    err = ctypes.c_uint32(0)
    st = int(_lib.alspec_get_device_error(workspace, workspace_bytes, stream, ctypes.byref(err)))
    return st, int(err.value)


def alspec_graph_begin(stream: int) -> int:
    return int(_lib.alspec_graph_begin(stream))


def alspec_graph_end(stream: int):
    g = ctypes.c_void_p(0)
    st = int(_lib.alspec_graph_end(stream, ctypes.byref(g)))
    return st, int(g.value or 0)


def alspec_graph_launch(graph: int, stream: int) -> int:
    return int(_lib.alspec_graph_launch(graph, stream))


def alspec_graph_destroy(graph: int) -> int:
    return int(_lib.alspec_graph_destroy(graph))


def alspec_shutdown() -> int:
    return int(_lib.alspec_shutdown())


def alspec_status_string(status: int) -> str:
    return _lib.alspec_status_string(int(status)).decode()


def alspec_version() -> int:
    return int(_lib.alspec_version())


def alspec_last_cuda_error() -> int:
    return int(_lib.alspec_last_cuda_error())


# ------------------------------------------------------------ torch layer

ENGINES = {"auto": ALSPEC_ENGINE_AUTO, "cuda_cores": ALSPEC_ENGINE_CUDA_CORES,
           "tensor_cores": ALSPEC_ENGINE_TENSOR_CORES}
SCHEDULES = {"auto": ALSPEC_SCHEDULE_AUTO, "streams": ALSPEC_SCHEDULE_STREAMS,
             "fused": ALSPEC_SCHEDULE_FUSED, "sink_first": ALSPEC_SCHEDULE_SINK_FIRST}


def make_desc(batch, n_q_heads, n_kv_heads, head_dim, max_seq_len, dtype, split_tokens=0,
              timeout_ms=0, engine="auto", schedule="auto") -> alspec_desc:
    code = {"bf16": ALSPEC_BF16, "f32": ALSPEC_F32}.get(dtype, dtype)
    eng = ENGINES.get(engine, engine)
    sch = SCHEDULES.get(schedule, schedule)
    return alspec_desc(batch, n_q_heads, n_kv_heads, head_dim, max_seq_len, int(code),
                       split_tokens, timeout_ms, int(eng), int(sch))


def _check(status: int, where: str):
    if status != ALSPEC_OK:
        raise AlspecError(status, where)


class Decoder:
    """One decode-attention shape with its own device workspace.

    ``decode`` takes device tensors (q [B, Hq, d], k/v [B, Hkv, Lmax, d] in
    bf16 or fp32, seq_lens int32 [B]) and returns (or fills) out_spec,
    out_exact (fp32 [B, Hq, d]), rel_l2 (fp32 [B]) and commit (uint8 [B]).
    """

    def __init__(self, batch, n_q_heads, n_kv_heads, head_dim, max_seq_len, dtype, n_sink,
                 window, device=None, split_tokens=0, timeout_ms=0, engine="auto",
                 schedule="auto"):
        import torch
        self.torch = torch
        self.desc = make_desc(batch, n_q_heads, n_kv_heads, head_dim, max_seq_len, dtype,
                              split_tokens, timeout_ms, engine, schedule)
        self.n_sink, self.window = int(n_sink), int(window)
        nbytes = alspec_workspace_size(self.desc, self.n_sink, self.window)
        if nbytes == 0:
            raise AlspecError(ALSPEC_ERR_INVALID_ARG, "alspec_workspace_size")
        self.device = torch.device(device) if device is not None else torch.device("cuda")
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        self.workspace_bytes = nbytes

    def plan(self):
        st, info = alspec_query_plan(self.desc, self.n_sink, self.window)
        _check(st, "alspec_query_plan")
        return info

    def alloc_outputs(self):
        t = self.torch
        d = self.desc
        kw = dict(device=self.device)
        return dict(out_spec=t.empty(d.batch, d.n_q_heads, d.head_dim, dtype=t.float32, **kw),
                    out_exact=t.empty(d.batch, d.n_q_heads, d.head_dim, dtype=t.float32, **kw),
                    rel_l2=t.empty(d.batch, dtype=t.float32, **kw),
                    commit=t.empty(d.batch, dtype=t.uint8, **kw))

    def decode(self, q, k, v, seq_lens, lam, out=None, stream=None, spec_event=None,
               prof_events=None, trace=None):
        """prof_events: None or ALSPEC_PROF_EVENTS torch.cuda.Event(enable_timing=True).
        trace: None or a zeroed int64 device tensor of 2 elements (see
        alspec_decode_traced); exclusive with the events."""
        t = self.torch
        out = out if out is not None else self.alloc_outputs()
        s = stream if stream is not None else t.cuda.current_stream(self.device)
        if trace is not None:
            if spec_event is not None or prof_events is not None:
                raise ValueError("trace excludes spec_event and prof_events")
            st = alspec_decode_traced(self.desc, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                      seq_lens.data_ptr(), self.n_sink, self.window, float(lam),
                                      out["out_spec"].data_ptr(), out["out_exact"].data_ptr(),
                                      out["rel_l2"].data_ptr(), out["commit"].data_ptr(),
                                      self.workspace.data_ptr(), self.workspace_bytes,
                                      s.cuda_stream, trace.data_ptr())
            _check(st, "alspec_decode_traced")
            return out
        ev = spec_event.cuda_event if spec_event is not None else 0
        prof = None
        if prof_events is not None:
            prof = [e.cuda_event for e in prof_events]
        if (spec_event is not None and not ev) or (prof is not None and not all(prof)):
            # torch creates the CUDA event lazily at its first record().
            raise ValueError("event has no CUDA handle yet: record() it once before passing it")
        st = alspec_decode(self.desc, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                           seq_lens.data_ptr(), self.n_sink, self.window, float(lam),
                           out["out_spec"].data_ptr(), out["out_exact"].data_ptr(),
                           out["rel_l2"].data_ptr(), out["commit"].data_ptr(),
                           self.workspace.data_ptr(), self.workspace_bytes, s.cuda_stream, ev,
                           prof)
        _check(st, "alspec_decode")
        return out

    def decode_oproj(self, q, k, v, seq_lens, lam, w_o, out=None, stream=None, trace=None,
                     gate="kernel"):
        """decode() plus y = o_proj(commit ? O_spec : O_exact) with w_o bf16
        [hidden, Hq * d]; out gains "y" (fp32 [B, hidden]).  trace: None or
        a zeroed int64 device tensor of 3 elements; gate: "kernel" or
        "graph_conditional"."""
        t = self.torch
        out = out if out is not None else self.alloc_outputs()
        hidden = int(w_o.shape[0])
        if "y" not in out:
            out["y"] = t.empty(self.desc.batch, hidden, dtype=t.float32, device=self.device)
        s = stream if stream is not None else t.cuda.current_stream(self.device)
        st = alspec_decode_oproj(self.desc, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                 seq_lens.data_ptr(), self.n_sink, self.window, float(lam),
                                 w_o.data_ptr(), hidden, out["out_spec"].data_ptr(),
                                 out["out_exact"].data_ptr(), out["rel_l2"].data_ptr(),
                                 out["commit"].data_ptr(), out["y"].data_ptr(), GATES[gate],
                                 self.workspace.data_ptr(), self.workspace_bytes, s.cuda_stream,
                                 trace.data_ptr() if trace is not None else 0)
        _check(st, "alspec_decode_oproj")
        return out

    def device_error(self, stream=None):
        t = self.torch
        s = stream if stream is not None else t.cuda.current_stream(self.device)
        return alspec_get_device_error(self.workspace.data_ptr(), self.workspace_bytes,
                                       s.cuda_stream)
