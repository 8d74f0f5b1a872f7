"""Python binding of libgpt.so, the B200 GPT pretraining-step library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/gpt.h.  PyTorch provides device
memory and the stream.  If the compiled library is missing the import of
``lib()`` raises; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgpt.so")

GPT_OK, GPT_EINVAL, GPT_ERANGE, GPT_ETIMEOUT, GPT_ECUDA = 0, -1, -2, -3, -4
KIND_PARAM, KIND_GRAD, KIND_MOM, KIND_ADAM_M, KIND_ADAM_V, KIND_NORMUON_V = 0, 1, 2, 3, 4, 5
REGION_MASTER, REGION_BF16, REGION_GRAD = 0, 1, 2
GROUP_ADAMW, GROUP_MUON = 0, 1
PROF_CATEGORIES = ["qkv_gemm", "proj_gemm", "fc_gemm", "down_gemm", "attn_fwd", "attn_bwd", "logits_gemm",
                   "ce_finish", "lm_dx_gemm", "lm_dw_gemm", "dx_gemm", "dw_gemm", "norm", "qk_bwd", "embed",
                   "ns_gemm", "muon_elem", "adamw", "fp8_quant"]

ABI_FUNCTIONS = [
    "gpt_workspace_size", "gpt_init", "gpt_fwd_bwd", "muon_step", "muon_step_normuon", "muon_step_layers",
    "gpt_block_region", "adamw_step", "gpt_train_step_host", "gpt_num_tensors", "gpt_tensor_info",
    "gpt_get_tensor", "gpt_set_tensor", "gpt_get_row_loss", "gpt_grad_region", "gpt_check",
    "gpt_launch_count", "gpt_profile_enable", "gpt_profile_read", "gpt_destroy", "gpt_last_error",
    "gpt_op_matmul_bf16", "gpt_op_matmul_tf32", "gpt_op_quantize_e4m3", "gpt_op_matmul_fp8",
    "gpt_op_attention_fwd", "gpt_op_attention_bwd", "gpt_op_attention_fwd_ex", "gpt_op_attention_bwd_ex",
    "gpt_op_rmsnorm_fwd", "gpt_op_newton_schulz_scratch", "gpt_op_newton_schulz",
    "gpt_op_newton_schulz_noalloc", "gpt_get_adam_step", "gpt_set_adam_step", "gpt_set_wait_limit",
    "gpt_op_check", "gpt_op_set_wait_limit", "gpt_op_embedding_bwd_scratch", "gpt_op_embedding_bwd",
    "adamw_step_shard", "gpt_tensor_region", "gpt_grad_bucket", "gpt_set_grad_events",
]
GRAD_BUCKETS = 6


class GptError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"libgpt error {code}: {msg}")
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [("depth", ctypes.c_int32), ("d_model", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("batch", ctypes.c_int32), ("seq_len", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("mlp_mult", ctypes.c_int32), ("precision", ctypes.c_int32), ("ns_tf32_steps", ctypes.c_int32),
                ("lm_chunk_rows", ctypes.c_int32), ("seed", ctypes.c_uint64), ("short_window", ctypes.c_int32),
                ("window_pattern", ctypes.c_char * 12), ("residual_extras", ctypes.c_int32),
                ("ve_gate_channels", ctypes.c_int32), ("n_kv_head", ctypes.c_int32)]


class HParams(ctypes.Structure):
    _fields_ = [("muon_lr", ctypes.c_float), ("muon_momentum", ctypes.c_float), ("muon_wd", ctypes.c_float),
                ("adam_lr", ctypes.c_float), ("adam_beta1", ctypes.c_float), ("adam_beta2", ctypes.c_float),
                ("adam_eps", ctypes.c_float), ("adam_wd", ctypes.c_float)]


_LIB = None


def lib():
    """The loaded library (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m gpt_pretraining_step_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        sig = {
            "gpt_workspace_size": (i32, [ctypes.POINTER(Config), ctypes.POINTER(sz), ctypes.POINTER(sz),
                                         ctypes.POINTER(sz)]),
            "gpt_init": (i32, [ctypes.POINTER(Config), vp, vp, vp, vp, ctypes.POINTER(vp)]),
            "gpt_fwd_bwd": (i32, [vp, vp, vp, vp, i32]),
            "muon_step": (i32, [vp, f32, f32, f32]),
            "muon_step_normuon": (i32, [vp, f32, f32, f32, f32]),
            "muon_step_layers": (i32, [vp, f32, f32, f32, f32, i32, i32]),
            "gpt_block_region": (i32, [vp, i32, i32, i32, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)]),
            "adamw_step": (i32, [vp, f32, f32, f32, f32, f32]),
            "adamw_step_shard": (i32, [vp, f32, f32, f32, f32, f32, i32, i32]),
            "gpt_tensor_region": (i32, [vp, i32, i32, i32, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)]),
            "gpt_grad_bucket": (i32, [vp, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)]),
            "gpt_set_grad_events": (i32, [vp, ctypes.POINTER(ctypes.c_void_p), i32]),
            "gpt_train_step_host": (i32, [vp, vp, vp, ctypes.POINTER(HParams), vp]),
            "gpt_num_tensors": (i32, [vp]),
            "gpt_tensor_info": (i32, [vp, i32, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32),
                                      ctypes.POINTER(ctypes.c_int32)]),
            "gpt_get_tensor": (i32, [vp, i32, i32, vp]),
            "gpt_set_tensor": (i32, [vp, i32, i32, vp]),
            "gpt_get_row_loss": (i32, [vp, vp]),
            "gpt_grad_region": (i32, [vp, ctypes.POINTER(sz), ctypes.POINTER(sz)]),
            "gpt_get_adam_step": (i32, [vp, ctypes.POINTER(ctypes.c_int64)]),
            "gpt_set_adam_step": (i32, [vp, ctypes.c_int64]),
            "gpt_check": (i32, [vp]),
            "gpt_set_wait_limit": (i32, [vp, ctypes.c_longlong]),
            "gpt_op_check": (i32, [vp]),
            "gpt_op_set_wait_limit": (i32, [ctypes.c_longlong]),
            "gpt_launch_count": (ctypes.c_int64, [vp]),
            "gpt_profile_enable": (i32, [vp, ctypes.c_uint32]),
            "gpt_profile_read": (i32, [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]),
            "gpt_destroy": (None, [vp]),
            "gpt_last_error": (ctypes.c_char_p, []),
            "gpt_op_matmul_bf16": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]),
            "gpt_op_matmul_tf32": (i32, [vp, vp, vp, i32, i32, i32, i32, vp]),
            "gpt_op_quantize_e4m3": (i32, [vp, ctypes.c_longlong, vp, vp, vp, vp]),
            "gpt_op_matmul_fp8": (i32, [vp, vp, vp, i32, i32, i32, vp, vp, i32, vp]),
            "gpt_op_attention_fwd": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, vp]),
            "gpt_op_attention_bwd": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp]),
            "gpt_op_attention_fwd_ex": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp]),
            "gpt_op_attention_bwd_ex": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp]),
            "gpt_op_rmsnorm_fwd": (i32, [vp, vp, vp, i32, i32, vp]),
            "gpt_op_embedding_bwd_scratch": (sz, [i32, i32]),
            "gpt_op_embedding_bwd": (i32, [vp, vp, vp, i32, i32, i32, i32, vp, vp]),
            "gpt_op_newton_schulz_scratch": (sz, [i32, i32, i32]),
            "gpt_op_newton_schulz": (i32, [vp, vp, i32, i32, i32, i32, vp, vp]),
            "gpt_op_newton_schulz_noalloc": (i32, [vp, vp, i32, i32, i32, i32, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _check(rc):
    if rc != GPT_OK:
        raise GptError(rc, lib().gpt_last_error().decode())
    return rc


def make_config(depth, batch, seq_len, vocab=32768, d_model=0, ns_tf32_steps=-1, lm_chunk_rows=0, seed=0,
                precision=0, window_pattern="", short_window=0, residual_extras=False, ve_gate_channels=0,
                n_kv_head=0):
    return Config(depth=depth, d_model=d_model, vocab=vocab, batch=batch, seq_len=seq_len, head_dim=128,
                  mlp_mult=4, precision=precision, ns_tf32_steps=ns_tf32_steps, lm_chunk_rows=lm_chunk_rows,
                  seed=seed, short_window=short_window, window_pattern=window_pattern.encode("ascii"),
                  residual_extras=int(bool(residual_extras)), ve_gate_channels=int(ve_gate_channels),
                  n_kv_head=int(n_kv_head))


def workspace_size(cfg: Config):
    p, s, a = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().gpt_workspace_size(ctypes.byref(cfg), ctypes.byref(p), ctypes.byref(s), ctypes.byref(a)))
    return p.value, s.value, a.value


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class GPTStep:
    """One GPT training-step context on the current CUDA device.

    The three workspace buffers are allocated with torch and owned by this
    object; every computation runs in libgpt's kernels on ``stream``.
    """

    def __init__(self, depth, batch, seq_len, vocab=32768, d_model=0, ns_tf32_steps=-1, lm_chunk_rows=0,
                 seed=0, stream=None, precision=0, window_pattern="", short_window=0, residual_extras=False,
                 ve_gate_channels=0, n_kv_head=0):
        import torch
        self.cfg = make_config(depth, batch, seq_len, vocab, d_model, ns_tf32_steps, lm_chunk_rows, seed, precision,
                               window_pattern, short_window, residual_extras, ve_gate_channels, n_kv_head)
        self.sizes = workspace_size(self.cfg)
        dev = torch.device("cuda", torch.cuda.current_device())
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self.bufs = [torch.empty(max(n, 256), dtype=torch.uint8, device=dev) for n in self.sizes]
        self.loss = torch.zeros(4, dtype=torch.float32, device=dev)
        h = ctypes.c_void_p()
        _check(lib().gpt_init(ctypes.byref(self.cfg), *[_ptr(b) for b in self.bufs], _stream(self.stream),
                              ctypes.byref(h)))
        self.h = h
        self.d_model = self.cfg.d_model or 64 * depth

    def __del__(self):
        h = getattr(self, "h", None)
        if h is not None and _LIB is not None:
            _LIB.gpt_destroy(h)
            self.h = None

    # -- the step
    def fwd_bwd(self, tokens, targets, accumulate=False, loss_out=None):
        out = self.loss if loss_out is None else loss_out
        _check(lib().gpt_fwd_bwd(self.h, _ptr(tokens), _ptr(targets), _ptr(out), int(bool(accumulate))))
        self._join_current_stream()
        return out[0] if loss_out is None else out

    def muon_step(self, lr=0.02, momentum=0.95, weight_decay=0.0):
        _check(lib().muon_step(self.h, lr, momentum, weight_decay))

    def muon_step_normuon(self, lr=0.02, momentum=0.95, weight_decay=0.0, beta2=0.95):
        _check(lib().muon_step_normuon(self.h, lr, momentum, weight_decay, beta2))

    def muon_step_layers(self, l0, l1, lr=0.02, momentum=0.95, weight_decay=0.0, normuon_beta2=-1.0):
        """Muon (or NorMuon with normuon_beta2 >= 0) of layers l0 .. l1-1 only."""
        _check(lib().muon_step_layers(self.h, lr, momentum, weight_decay, normuon_beta2, int(l0), int(l1)))

    def block_region(self, what, kind, l0, l1):
        """Tensor view of block matrix kind (0 q|k|v, 1 attention output, 2 MLP
        up, 3 MLP down) for layers l0 .. l1-1: REGION_MASTER (fp32), REGION_BF16
        (bf16 working copies) or REGION_GRAD (fp32 gradients)."""
        import torch
        off, n = ctypes.c_size_t(), ctypes.c_size_t()
        _check(lib().gpt_block_region(self.h, int(what), int(kind), int(l0), int(l1), ctypes.byref(off),
                                      ctypes.byref(n)))
        buf = self.bufs[1] if what == REGION_GRAD else self.bufs[0]
        return buf[off.value:off.value + n.value].view(torch.bfloat16 if what == REGION_BF16 else torch.float32)

    def adamw_grad_view(self):
        """fp32 gradients of the token embedding and lm_head (the part of the
        gradient span before the block matrices)."""
        import torch
        off, n = ctypes.c_size_t(), ctypes.c_size_t()
        _check(lib().gpt_grad_region(self.h, ctypes.byref(off), ctypes.byref(n)))
        first, size = ctypes.c_size_t(), ctypes.c_size_t()
        _check(lib().gpt_block_region(self.h, REGION_GRAD, 0, 0, 0, ctypes.byref(first), ctypes.byref(size)))
        return self.bufs[1][off.value:first.value].view(torch.float32)

    def adamw_step(self, lr=3e-3, beta1=0.8, beta2=0.95, eps=1e-10, weight_decay=0.0):
        _check(lib().adamw_step(self.h, lr, beta1, beta2, eps, weight_decay))

    def adamw_step_shard(self, part, nparts, lr=3e-3, beta1=0.8, beta2=0.95, eps=1e-10, weight_decay=0.0):
        """AdamW on share `part` of `nparts` of the embedding and lm_head rows
        (the other AdamW tensors whole)."""
        _check(lib().adamw_step_shard(self.h, lr, beta1, beta2, eps, weight_decay, int(part), int(nparts)))

    def tensor_region(self, what, tid, row0, row1):
        """Tensor view of rows row0 .. row1-1 of tensor tid (embedding, lm_head or
        a block matrix): REGION_MASTER, REGION_BF16 or REGION_GRAD."""
        import torch
        off, n = ctypes.c_size_t(), ctypes.c_size_t()
        _check(lib().gpt_tensor_region(self.h, int(what), int(tid), int(row0), int(row1), ctypes.byref(off),
                                       ctypes.byref(n)))
        buf = self.bufs[1] if what == REGION_GRAD else self.bufs[0]
        return buf[off.value:off.value + n.value].view(torch.bfloat16 if what == REGION_BF16 else torch.float32)

    def grad_bucket(self, i):
        """fp32 view of gradient bucket i (see gpt_grad_bucket)."""
        import torch
        off, n = ctypes.c_size_t(), ctypes.c_size_t()
        _check(lib().gpt_grad_bucket(self.h, int(i), ctypes.byref(off), ctypes.byref(n)))
        return self.bufs[1][off.value:off.value + n.value].view(torch.float32)

    def set_grad_events(self, events):
        """Register torch.cuda.Event objects: events[i] is recorded on the
        context's stream when gradient bucket i is complete (empty: stop)."""
        self._grad_events = list(events)   # kept alive while registered
        handles = []
        for e in self._grad_events:
            e.record(self.stream)           # creates the event on this device
            handles.append(ctypes.c_void_p(e.cuda_event))
        arr = (ctypes.c_void_p * max(1, len(handles)))(*handles)
        _check(lib().gpt_set_grad_events(self.h, arr, len(handles)))

    def train_step_host(self, tokens_host, targets_host, hp: HParams):
        """Whole step from host int32 arrays (numpy or pinned torch); returns the loss."""
        loss = ctypes.c_float()
        tp = tokens_host.ctypes.data if hasattr(tokens_host, "ctypes") else tokens_host.data_ptr()
        gp = targets_host.ctypes.data if hasattr(targets_host, "ctypes") else targets_host.data_ptr()
        _check(lib().gpt_train_step_host(self.h, ctypes.c_void_p(tp), ctypes.c_void_p(gp), ctypes.byref(hp),
                                         ctypes.byref(loss)))
        return loss.value

    # -- tensors
    def num_tensors(self):
        return lib().gpt_num_tensors(self.h)

    def tensor_info(self, tid):
        r, c, g = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib().gpt_tensor_info(self.h, tid, ctypes.byref(r), ctypes.byref(c), ctypes.byref(g)))
        return r.value, c.value, g.value

    def _shape(self, tid, kind):
        r, c, _ = self.tensor_info(tid)
        return (self.d_model,) if kind == KIND_NORMUON_V else (r, c)

    def get(self, tid, kind=KIND_PARAM):
        """A copy of the tensor, ordered before later work on torch's current
        stream (the copy runs on the context's stream)."""
        import torch
        out = torch.empty(self._shape(tid, kind), dtype=torch.float32, device=self.bufs[0].device)
        _check(lib().gpt_get_tensor(self.h, tid, kind, _ptr(out)))
        self._join_current_stream()
        return out

    def _join_current_stream(self):
        # work queued on the context's stream (a copy into a torch tensor)
        # completes before anything torch's current stream runs next
        import torch
        cur = torch.cuda.current_stream(self.bufs[0].device)
        if cur.cuda_stream != self.stream.cuda_stream:
            cur.wait_stream(self.stream)

    def set(self, tid, value, kind=KIND_PARAM):
        import torch
        shape = self._shape(tid, kind)
        v = torch.as_tensor(value, dtype=torch.float32).to(self.bufs[0].device).contiguous()
        if tuple(v.shape) != shape:
            raise ValueError(f"tensor {tid} has shape {shape}, got {tuple(v.shape)}")
        _check(lib().gpt_set_tensor(self.h, tid, kind, _ptr(v)))
        self.stream.synchronize()

    def grad_view(self):
        """fp32 view of every gradient (one span of the state buffer), e.g. for an all-reduce."""
        import torch
        off, n = ctypes.c_size_t(), ctypes.c_size_t()
        _check(lib().gpt_grad_region(self.h, ctypes.byref(off), ctypes.byref(n)))
        return self.bufs[1][off.value:off.value + n.value].view(torch.float32)

    def row_loss(self):
        import torch
        out = torch.empty((self.cfg.batch, self.cfg.seq_len), dtype=torch.float32, device=self.bufs[0].device)
        _check(lib().gpt_get_row_loss(self.h, _ptr(out)))
        self._join_current_stream()
        return out

    def check(self):
        return _check(lib().gpt_check(self.h))

    def set_wait_limit(self, cycles):
        """Bound of the kernels' device-side waits in SM cycles (<= 0: the default)."""
        _check(lib().gpt_set_wait_limit(self.h, int(cycles)))

    # -- checkpoint
    def _state_kinds(self, tid):
        _, _, group = self.tensor_info(tid)
        if group == GROUP_MUON:
            return (KIND_PARAM, KIND_MOM, KIND_NORMUON_V)
        return (KIND_PARAM, KIND_ADAM_M, KIND_ADAM_V)

    def state_dict(self):
        """Every tensor's value and optimizer state (host float32 arrays, keyed
        (tensor id, kind)) and the AdamW step count: what a checkpoint needs."""
        step = ctypes.c_int64()
        _check(lib().gpt_get_adam_step(self.h, ctypes.byref(step)))
        tensors = {}
        for tid in range(self.num_tensors()):
            for kind in self._state_kinds(tid):
                tensors[(tid, kind)] = self.get(tid, kind).cpu().numpy()
        return {"tensors": tensors, "adam_step": int(step.value)}

    def load_state_dict(self, state):
        """Restore what state_dict returned (same configuration)."""
        for (tid, kind), value in state["tensors"].items():
            self.set(tid, value, kind)
        _check(lib().gpt_set_adam_step(self.h, int(state["adam_step"])))

    def launch_count(self):
        return lib().gpt_launch_count(self.h)

    def profile_enable(self, categories):
        """Record events around the launches of the named categories (empty = off)."""
        mask = 0
        for c in categories:
            mask |= 1 << PROF_CATEGORIES.index(c)
        _check(lib().gpt_profile_enable(self.h, mask))

    def profile_read(self):
        """{category: (ms, launches)} since the last read (synchronises)."""
        n = len(PROF_CATEGORIES)
        ms = (ctypes.c_double * n)()
        cnt = (ctypes.c_int64 * n)()
        _check(lib().gpt_profile_read(self.h, ms, cnt))
        return {PROF_CATEGORIES[i]: (ms[i], cnt[i]) for i in range(n) if cnt[i]}


# ---------------------------------------------------------------- op level

def op_check(stream=None):
    """Synchronise the stream and raise GptError (GPT_ETIMEOUT) if a bounded
    device wait of an op-level call expired since the last check."""
    return _check(lib().gpt_op_check(_stream(stream)))


def op_set_wait_limit(cycles):
    """Bound of the device-side waits of later op-level calls (<= 0: default)."""
    _check(lib().gpt_op_set_wait_limit(int(cycles)))


def matmul_bf16(A, B, M, N, K, batch=1, a_trans=False, b_trans=False, out=None, stream=None):
    import torch
    C = out if out is not None else torch.empty((batch, M, N), dtype=torch.float32, device=A.device)
    _check(lib().gpt_op_matmul_bf16(_ptr(A), _ptr(B), _ptr(C), M, N, K, batch, int(a_trans), int(b_trans),
                                    _stream(stream)))
    return C


def matmul_tf32(A, B, M, N, K, b_trans=False, stream=None):
    import torch
    C = torch.empty((M, N), dtype=torch.float32, device=A.device)
    _check(lib().gpt_op_matmul_tf32(_ptr(A), _ptr(B), _ptr(C), M, N, K, int(b_trans), _stream(stream)))
    return C


def quantize_e4m3(x, stream=None):
    """(q uint8 tensor of e4m3 codes, inv scale tensor) for a bf16 tensor x."""
    import torch
    q = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    inv = torch.empty(1, dtype=torch.float32, device=x.device)
    amax = torch.empty(1, dtype=torch.int32, device=x.device)
    _check(lib().gpt_op_quantize_e4m3(_ptr(x), x.numel(), _ptr(q), _ptr(inv), _ptr(amax), _stream(stream)))
    return q.view(x.shape), inv


def matmul_fp8(A, B, M, N, K, inv_a, inv_b, b_trans=False, stream=None):
    import torch
    C = torch.empty((M, N), dtype=torch.float32, device=A.device)
    _check(lib().gpt_op_matmul_fp8(_ptr(A), _ptr(B), _ptr(C), M, N, K, _ptr(inv_a), _ptr(inv_b), int(b_trans),
                                   _stream(stream)))
    return C


def attention_fwd(q, k, v, window=-1, stream=None):
    """Causal attention; k, v may have fewer heads than q (grouped kv heads);
    window >= 0 limits query t to keys t - window .. t."""
    import torch
    B, H, T, hd = q.shape
    Hkv = k.shape[1]
    o = torch.empty((B, T, H, hd), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    _check(lib().gpt_op_attention_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, T, int(window),
                                         _stream(stream)))
    return o, lse


def attention_bwd(q, k, v, o, lse, dout, window=-1, stream=None):
    import torch
    B, H, T, hd = q.shape
    Hkv = k.shape[1]
    dq = torch.empty((B, H, T, hd), dtype=torch.float32, device=q.device)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    D = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    _check(lib().gpt_op_attention_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(D),
                                         _ptr(dq), _ptr(dk), _ptr(dv), B, H, Hkv, T, int(window), _stream(stream)))
    return dq, dk, dv


def rmsnorm_fwd(x, stream=None):
    import torch
    M, d = x.shape
    y = torch.empty((M, d), dtype=torch.bfloat16, device=x.device)
    r = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check(lib().gpt_op_rmsnorm_fwd(_ptr(x), _ptr(y), _ptr(r), M, d, _stream(stream)))
    return y, r


def embedding_bwd(tokens, dx, vocab, dwte=None, accumulate=False, stream=None):
    """dwte [vocab, d] (+)= rows of dx [M, d] scattered by token (int32 [M])."""
    import torch
    M, d = dx.shape
    out = torch.zeros((vocab, d), dtype=torch.float32, device=dx.device) if dwte is None else dwte
    scratch = torch.empty(max(lib().gpt_op_embedding_bwd_scratch(M, d), 256), dtype=torch.uint8, device=dx.device)
    _check(lib().gpt_op_embedding_bwd(_ptr(tokens), _ptr(dx), _ptr(out), M, d, vocab, int(bool(accumulate)),
                                      _ptr(scratch), _stream(stream)))
    return out


def newton_schulz(G, tf32_steps=-1, stream=None):
    import torch
    batch, rows, cols = G.shape
    X = torch.empty_like(G)
    n = lib().gpt_op_newton_schulz_scratch(batch, rows, cols)
    scratch = torch.empty(n, dtype=torch.uint8, device=G.device)
    _check(lib().gpt_op_newton_schulz(_ptr(G), _ptr(X), batch, rows, cols, tf32_steps, _ptr(scratch),
                                      _stream(stream)))
    return X


def newton_schulz_noalloc(G, tf32_steps=-1, X=None, stream=None):
    """Newton-Schulz through the entry point that allocates no device memory.

    The library keeps the scratch in its own fixed device array (at most
    batch * rows * cols = 262144 elements); only the output is caller memory.
    Calls that overlap on the GPU share that array and must not run
    concurrently.
    """
    import torch
    batch, rows, cols = G.shape
    X = torch.empty_like(G) if X is None else X
    _check(lib().gpt_op_newton_schulz_noalloc(_ptr(G), _ptr(X), batch, rows, cols, tf32_steps, _stream(stream)))
    return X
