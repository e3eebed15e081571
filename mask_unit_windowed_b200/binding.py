"""Thin Python binding of libhiera.so (include/hiera.h): argument marshalling only.

Every step of the Hiera block runs inside the library's CUDA kernels. PyTorch supplies
device memory (outputs, workspaces, packed weights) and the current CUDA stream; the
calls below pass raw pointers and sizes through ctypes and raise HieraError on any
non-OK status. If libhiera.so has not been built the import of `lib()` fails loudly:
there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhiera.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "hiera.h")

HIERA_F32, HIERA_BF16 = 0, 1
STATUS = {0: "HIERA_OK", 1: "HIERA_ERR_INVALID_ARG", 2: "HIERA_ERR_SHAPE", 3: "HIERA_ERR_DTYPE",
          4: "HIERA_ERR_ALIGNMENT", 5: "HIERA_ERR_WORKSPACE", 6: "HIERA_ERR_CUDA",
          7: "HIERA_ERR_TIMEOUT", 8: "HIERA_ERR_DEVICE"}
PATCH_PACKED_BYTES = (196 * 112 + 112) * 4 + 112 * 208 * 2


class HieraError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


class BlockDescC(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("tokens", ctypes.c_int), ("dim_in", ctypes.c_int),
                ("dim_out", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("q_stride", ctypes.c_int), ("window_tokens", ctypes.c_int),
                ("mask_unit_attn", ctypes.c_int), ("ln_eps", ctypes.c_float),
                ("dtype", ctypes.c_int)]


WEIGHT_NAMES = ("norm1_w", "norm1_b", "qkv_w", "qkv_b", "proj_w", "proj_b", "attn_proj_w",
                "attn_proj_b", "norm2_w", "norm2_b", "fc1_w", "fc1_b", "fc2_w", "fc2_b")


class BlockWeightsC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_NAMES]


class BackboneDescC(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("img", ctypes.c_int),
                ("mask_unit_attn_stage2_first", ctypes.c_int), ("dtype", ctypes.c_int)]


class BackboneWeightsC(ctypes.Structure):
    _fields_ = [("patch_w", ctypes.c_void_p), ("patch_b", ctypes.c_void_p),
                ("pos_embed", ctypes.c_void_p), ("blocks", BlockWeightsC * 24)]


_lib = None


def header_symbols() -> list:
    """Names of every entry point declared in include/hiera.h."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"HIERA_API\s+[\w\s\*]+?\b(hiera_\w+)\s*\(", text)


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m mask_unit_windowed_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        sig = {
            "hiera_status_string": ([I], ctypes.c_char_p),
            "hiera_get_device_status": ([P], I),
            "hiera_unroll": ([P, P, I, I, I, I, I, P], I),
            "hiera_reroll": ([P, P, I, I, I, I, I, P], I),
            "hiera_linear": ([P, P, P, P, P, I, I, I, I, P], I),
            "hiera_block_packed_bytes": ([ctypes.POINTER(BlockDescC)], S),
            "hiera_block_pack": ([ctypes.POINTER(BlockDescC), ctypes.POINTER(BlockWeightsC), P, S,
                                  P], I),
            "hiera_block_workspace_bytes": ([ctypes.POINTER(BlockDescC)], S),
            "hiera_block_forward": ([ctypes.POINTER(BlockDescC), P, P, P, P, S, P], I),
            "hiera_block_workspace_layout": ([ctypes.POINTER(BlockDescC),
                                              ctypes.POINTER(ctypes.c_longlong)], I),
            "hiera_patch_pack": ([P, P, P, I, P], I),
            "hiera_patch_embed": ([P, P, P, P, I, I, I, P], I),
            "hiera_backbone_packed_bytes": ([ctypes.POINTER(BackboneDescC)], S),
            "hiera_backbone_pack": ([ctypes.POINTER(BackboneDescC),
                                     ctypes.POINTER(BackboneWeightsC), P, S, P], I),
            "hiera_backbone_workspace_bytes": ([ctypes.POINTER(BackboneDescC)], S),
            "hiera_backbone_forward": ([ctypes.POINTER(BackboneDescC), P, P,
                                        ctypes.POINTER(ctypes.c_void_p), P, S, P], I),
            "hiera_debug_timeout_probe": ([I, P], I),
            "hiera_debug_gelu": ([P, P, I, P], I),
            "hiera_block_forward_noalloc": ([ctypes.POINTER(BlockDescC), P, P, P, P], I),
            "hiera_static_scratch_bytes": ([], S),
            "hiera_attention": ([P, P, P, P, I, I, I, I, I, P], I),
            "hiera_profile_begin": ([ctypes.POINTER(ctypes.c_void_p), I,
                                     ctypes.POINTER(ctypes.c_int)], I),
            "hiera_profile_end": ([P], I),
            "hiera_kernel_name": ([I], ctypes.c_char_p),
            "hiera_set_option": ([I, I], I),
            "hiera_get_option": ([I], I),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        del F
        _lib = L
    return _lib


def _check(code: int, where: str):
    if code != 0:
        raise HieraError(code, where)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HIERA_BF16
    if t.dtype == torch.float32:
        return HIERA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def _expect(t: torch.Tensor, name: str, shape, dtype, device=None):
    """Reject a tensor whose shape, dtype or device differs from what the C call will
    assume: the library sizes every copy from the descriptor alone, so a mismatched
    tensor would be read or written past its end."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    _need(t, name)
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _expect_bytes(t: torch.Tensor, name: str, nbytes: int, device=None):
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise ValueError(f"{name} holds {have} bytes, needs {nbytes}")
    _need(t, name)
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


# ----------------------------------------------------------------------------- Unroll / Reroll
def unroll(x: torch.Tensor, G: int, levels: int, out=None, stream=None) -> torch.Tensor:
    B, N, C = x.shape
    if N != G * G:
        raise ValueError(f"x has shape {tuple(x.shape)}: {N} tokens, expected G*G = {G * G}")
    _need(x, "x")
    out = torch.empty_like(x) if out is None else out
    _expect_bytes(out, "out", x.numel() * x.element_size(), x.device)
    _check(lib().hiera_unroll(_ptr(x), _ptr(out), B, G, C, levels, _dt(x), _stream(stream)),
           "hiera_unroll")
    return out


def reroll(x: torch.Tensor, G: int, levels: int, out=None, stream=None) -> torch.Tensor:
    B, N, C = x.shape
    if N != G * G:
        raise ValueError(f"x has shape {tuple(x.shape)}: {N} tokens, expected G*G = {G * G}")
    _need(x, "x")
    out = torch.empty((B, G, G, C), dtype=x.dtype, device=x.device) if out is None else out
    _expect_bytes(out, "out", x.numel() * x.element_size(), x.device)
    _check(lib().hiera_reroll(_ptr(x), _ptr(out), B, G, C, levels, _dt(x), _stream(stream)),
           "hiera_reroll")
    return out


def linear(x, w, bias=None, residual=None, out=None, stream=None) -> torch.Tensor:
    M, K = x.shape
    N = w.shape[0]
    if tuple(w.shape) != (N, K):
        raise ValueError(f"w has shape {tuple(w.shape)}, expected {(N, K)}")
    _need(x, "x")
    _expect(w, "w", (N, K), x.dtype, x.device)
    if bias is not None:
        _expect(bias, "bias", (N,), x.dtype, x.device)
    if residual is not None:
        _expect(residual, "residual", (M, N), x.dtype, x.device)
    out = torch.empty((M, N), dtype=x.dtype, device=x.device) if out is None else out
    _expect(out, "out", (M, N), x.dtype, x.device)
    _check(lib().hiera_linear(_ptr(x), _ptr(w), _ptr(bias), _ptr(residual), _ptr(out), M, N, K,
                              _dt(x), _stream(stream)), "hiera_linear")
    return out


# ----------------------------------------------------------------------------- block
@dataclass
class BlockDesc:
    B: int
    tokens: int
    dim_in: int
    dim_out: int
    heads: int
    q_stride: int = 1
    window_tokens: int = 64
    mask_unit_attn: bool = True
    dtype: torch.dtype = torch.bfloat16
    head_dim: int = 56
    ln_eps: float = 1e-6

    def c(self) -> BlockDescC:
        return BlockDescC(self.B, self.tokens, self.dim_in, self.dim_out, self.heads,
                          self.head_dim, self.q_stride, self.window_tokens,
                          int(bool(self.mask_unit_attn)), self.ln_eps,
                          HIERA_BF16 if self.dtype == torch.bfloat16 else HIERA_F32)

    @property
    def out_tokens(self) -> int:
        return self.tokens // self.q_stride


def _weights_c(w: dict) -> BlockWeightsC:
    wc = BlockWeightsC()
    for n in WEIGHT_NAMES:
        t = w.get(n)
        if t is not None:
            _need(t, n)
        setattr(wc, n, None if t is None else t.data_ptr())
    return wc


def block_packed_bytes(desc: BlockDesc) -> int:
    d = desc.c()
    n = lib().hiera_block_packed_bytes(ctypes.byref(d))
    if n == 0:
        raise HieraError(2, "hiera_block_packed_bytes")
    return n


def block_workspace_bytes(desc: BlockDesc) -> int:
    d = desc.c()
    n = lib().hiera_block_workspace_bytes(ctypes.byref(d))
    if n == 0:
        raise HieraError(2, "hiera_block_workspace_bytes")
    return n


def block_workspace_layout(desc: BlockDesc) -> list:
    d = desc.c()
    offs = (ctypes.c_longlong * 7)()
    _check(lib().hiera_block_workspace_layout(ctypes.byref(d), offs),
           "hiera_block_workspace_layout")
    return list(offs)


def block_pack(desc: BlockDesc, weights: dict, device="cuda", stream=None) -> torch.Tensor:
    d = desc.c()
    nbytes = block_packed_bytes(desc)
    packed = torch.empty(nbytes, dtype=torch.uint8, device=device)
    wc = _weights_c(weights)
    _check(lib().hiera_block_pack(ctypes.byref(d), ctypes.byref(wc), _ptr(packed), nbytes,
                                  _stream(stream)), "hiera_block_pack")
    return packed


def _check_block_args(desc: BlockDesc, packed, x, out):
    """Shapes, dtypes and devices of a block call against its descriptor (before any
    launch): every shape first, then where the tensors live."""
    out_shape = (desc.B, desc.out_tokens, desc.dim_out)
    for t, name, shape in ((x, "x", (desc.B, desc.tokens, desc.dim_in)), (out, "out", out_shape)):
        if t is not None and (tuple(t.shape) != shape or t.dtype != desc.dtype):
            raise ValueError(f"{name} is {tuple(t.shape)} {t.dtype}, expected {shape} "
                             f"{desc.dtype}: shape or dtype mismatch")
    _expect(x, "x", (desc.B, desc.tokens, desc.dim_in), desc.dtype)
    _expect_bytes(packed, "packed", block_packed_bytes(desc), x.device)
    if out is not None:
        _expect(out, "out", out_shape, desc.dtype, x.device)


def block_forward(desc: BlockDesc, packed: torch.Tensor, x: torch.Tensor, out=None,
                  workspace=None, stream=None) -> torch.Tensor:
    _check_block_args(desc, packed, x, out)
    d = desc.c()
    if out is None:
        out = torch.empty((desc.B, desc.out_tokens, desc.dim_out), dtype=x.dtype,
                          device=x.device)
    if workspace is None:
        workspace = torch.empty(block_workspace_bytes(desc), dtype=torch.uint8, device=x.device)
    _expect_bytes(workspace, "workspace", block_workspace_bytes(desc), x.device)
    _check(lib().hiera_block_forward(ctypes.byref(d), _ptr(packed), _ptr(x), _ptr(out),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream)),
           "hiera_block_forward")
    return out


def static_scratch_bytes() -> int:
    """Size of the library's static scratch array (hiera_static_scratch_bytes)."""
    return int(lib().hiera_static_scratch_bytes())


def block_forward_noalloc(desc: BlockDesc, packed: torch.Tensor, x: torch.Tensor, out=None,
                          stream=None) -> torch.Tensor:
    """hiera_block_forward_noalloc: the block forward with the library's static scratch
    (for callers that cannot allocate a workspace); `out` may be preallocated."""
    _check_block_args(desc, packed, x, out)
    d = desc.c()
    if out is None:
        out = torch.empty((desc.B, desc.out_tokens, desc.dim_out), dtype=x.dtype,
                          device=x.device)
    _check(lib().hiera_block_forward_noalloc(ctypes.byref(d), _ptr(packed), _ptr(x), _ptr(out),
                                             _stream(stream)), "hiera_block_forward_noalloc")
    return out


# ----------------------------------------------------------------------------- attention core
def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out=None,
              stream=None) -> torch.Tensor:
    """hiera_attention on head-major q [B, windows, heads, Tq, 64], k and v
    [B, windows, heads, Tkv, 64] (bf16; q/k channels 56..63 zero, v channel 56 = 1 and
    57..63 zero). Returns the merged [B, Tq * windows, heads * 56] output."""
    if q.dim() != 5 or k.dim() != 5:
        raise ValueError("q, k, v must be [B, windows, heads, T, 64]")
    B, nW, heads, Tq, _ = q.shape
    Tkv = k.shape[3]
    for t, name, T in ((q, "q", Tq), (k, "k", Tkv), (v, "v", Tkv)):
        if tuple(t.shape) != (B, nW, heads, T, 64) or t.dtype != torch.bfloat16:
            raise ValueError(f"{name} is {tuple(t.shape)} {t.dtype}: shape or dtype mismatch "
                             f"(expected {(B, nW, heads, T, 64)} bf16)")
    _expect(q, "q", (B, nW, heads, Tq, 64), torch.bfloat16)
    _expect(k, "k", (B, nW, heads, Tkv, 64), torch.bfloat16, q.device)
    _expect(v, "v", (B, nW, heads, Tkv, 64), torch.bfloat16, q.device)
    shape = (B, Tq * nW, heads * 56)
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=q.device)
    _expect(out, "out", shape, torch.bfloat16, q.device)
    _check(lib().hiera_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, nW, heads, Tq, Tkv,
                                 _stream(stream)), "hiera_attention")
    return out


# ----------------------------------------------------------------------------- patch embed
def patch_pack(patch_w, patch_b=None, stream=None) -> torch.Tensor:
    _need(patch_w, "patch_w")
    packed = torch.empty(PATCH_PACKED_BYTES, dtype=torch.uint8, device=patch_w.device)
    _check(lib().hiera_patch_pack(_ptr(patch_w), _ptr(patch_b), _ptr(packed), _dt(patch_w),
                                  _stream(stream)), "hiera_patch_pack")
    return packed


def patch_embed(img, packed_patch, pos_embed, out=None, stream=None) -> torch.Tensor:
    _need(img, "img")
    B, H, W, _ = img.shape
    G = H // 4
    _expect(img, "img", (B, H, H, 4), img.dtype)
    _expect_bytes(packed_patch, "packed_patch", PATCH_PACKED_BYTES, img.device)
    _expect(pos_embed, "pos_embed", (G * G, 112), img.dtype, img.device)
    out = torch.empty((B, G * G, 112), dtype=img.dtype, device=img.device) if out is None else out
    _expect(out, "out", (B, G * G, 112), img.dtype, img.device)
    _check(lib().hiera_patch_embed(_ptr(img), _ptr(packed_patch), _ptr(pos_embed), _ptr(out), B,
                                   H, _dt(img), _stream(stream)), "hiera_patch_embed")
    return out


# ----------------------------------------------------------------------------- backbone
@dataclass
class BackboneDesc:
    B: int
    img: int
    dtype: torch.dtype = torch.bfloat16
    mask_unit_attn_stage2_first: bool = False

    def c(self) -> BackboneDescC:
        return BackboneDescC(self.B, self.img, int(bool(self.mask_unit_attn_stage2_first)),
                             HIERA_BF16 if self.dtype == torch.bfloat16 else HIERA_F32)

    def feature_shapes(self):
        dims = (112, 224, 448, 896)
        return [(self.B, self.img >> (s + 2), self.img >> (s + 2), dims[s]) for s in range(4)]


def backbone_packed_bytes(desc: BackboneDesc) -> int:
    d = desc.c()
    n = lib().hiera_backbone_packed_bytes(ctypes.byref(d))
    if n == 0:
        raise HieraError(2, "hiera_backbone_packed_bytes")
    return n


def backbone_workspace_bytes(desc: BackboneDesc) -> int:
    d = desc.c()
    n = lib().hiera_backbone_workspace_bytes(ctypes.byref(d))
    if n == 0:
        raise HieraError(2, "hiera_backbone_workspace_bytes")
    return n


def backbone_pack(desc: BackboneDesc, weights: dict, device="cuda", stream=None) -> torch.Tensor:
    d = desc.c()
    wc = BackboneWeightsC()
    wc.patch_w = weights["patch_w"].data_ptr()
    wc.patch_b = None if weights.get("patch_b") is None else weights["patch_b"].data_ptr()
    wc.pos_embed = weights["pos_embed"].data_ptr()
    for i, bw in enumerate(weights["blocks"]):
        wc.blocks[i] = _weights_c(bw)
    nbytes = backbone_packed_bytes(desc)
    packed = torch.empty(nbytes, dtype=torch.uint8, device=device)
    _check(lib().hiera_backbone_pack(ctypes.byref(d), ctypes.byref(wc), _ptr(packed), nbytes,
                                     _stream(stream)), "hiera_backbone_pack")
    return packed


def backbone_forward(desc: BackboneDesc, packed, img, feats=None, workspace=None,
                     stream=None):
    _expect(img, "img", (desc.B, desc.img, desc.img, 4), desc.dtype)
    _expect_bytes(packed, "packed", backbone_packed_bytes(desc), img.device)
    d = desc.c()
    if feats is None:
        feats = [torch.empty(s, dtype=img.dtype, device=img.device)
                 for s in desc.feature_shapes()]
    if len(feats) != 4:
        raise ValueError("feats must hold four tensors")
    for i, (f, shp) in enumerate(zip(feats, desc.feature_shapes())):
        _expect(f, f"feats[{i}]", shp, desc.dtype, img.device)
    if workspace is None:
        workspace = torch.empty(backbone_workspace_bytes(desc), dtype=torch.uint8,
                                device=img.device)
    _expect_bytes(workspace, "workspace", backbone_workspace_bytes(desc), img.device)
    fp = (ctypes.c_void_p * 4)(*[f.data_ptr() for f in feats])
    _check(lib().hiera_backbone_forward(ctypes.byref(d), _ptr(packed), _ptr(img), fp,
                                        _ptr(workspace), workspace.numel() * workspace.element_size(),
                                        _stream(stream)),
           "hiera_backbone_forward")
    return feats


class BackbonePipeline:
    """Host-to-host inference over consecutive batches on one device.

    For each batch: upload the image from pinned host memory, run hiera_backbone_forward,
    download the four features into pinned host memory. Uploads, the forward calls and
    downloads go to three streams with two device buffer sets, so the copies of a batch
    overlap the compute of its neighbours; the forwards themselves run one after another on
    the compute stream (they share one workspace). With graph=True (the default) each
    buffer set's hiera_backbone_forward call is captured once in a CUDA graph and replayed,
    so the host does not re-enqueue its launches for every batch.

        pipe = BackbonePipeline(desc, packed)
        pipe.run(host_images, host_features)   # lists of pinned CPU tensors, one per batch
        pipe.synchronize()
    """

    def __init__(self, desc: BackboneDesc, packed: torch.Tensor, device=None, graph=True):
        self.desc, self.packed = desc, packed
        self.graph = graph
        self._graphs = [None, None]
        dev = packed.device if device is None else torch.device(device)
        shape = (desc.B, desc.img, desc.img, 4)
        self.imgs = [torch.empty(shape, dtype=desc.dtype, device=dev) for _ in range(2)]
        self.feats = [[torch.empty(s, dtype=desc.dtype, device=dev)
                       for s in desc.feature_shapes()] for _ in range(2)]
        self.ws = torch.empty(backbone_workspace_bytes(desc), dtype=torch.uint8, device=dev)
        self.s_in = torch.cuda.Stream(device=dev)
        self.s_comp = torch.cuda.Stream(device=dev)
        self.s_out = torch.cuda.Stream(device=dev)
        self._ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "comp", "out")}
        self._count = 0

    def host_feature_buffers(self):
        """A set of pinned host tensors shaped like one batch's features."""
        return [torch.empty(s, dtype=self.desc.dtype, pin_memory=True)
                for s in self.desc.feature_shapes()]

    def run(self, host_images, host_features, start_event=None, end_event=None):
        """Enqueue one upload / forward / download per batch. host_features[k] receives the
        features of host_images[k] (the same set may be passed for several batches: the
        downloads are ordered). Returns without waiting; see synchronize()."""
        ev_in, ev_comp, ev_out = self._ev["in"], self._ev["comp"], self._ev["out"]
        if start_event is not None:
            start_event.record(self.s_in)
        for h_img, h_feats in zip(host_images, host_features):
            i = self._count % 2
            if self._count >= 2:
                self.s_in.wait_event(ev_comp[i])    # device image buffer i is free again
            with torch.cuda.stream(self.s_in):
                self.imgs[i].copy_(h_img, non_blocking=True)
            ev_in[i].record(self.s_in)
            self.s_comp.wait_event(ev_in[i])
            if self._count >= 2:
                self.s_comp.wait_event(ev_out[i])   # feature buffers i were downloaded
            if not self.graph:
                backbone_forward(self.desc, self.packed, self.imgs[i], feats=self.feats[i],
                                 workspace=self.ws, stream=self.s_comp)
            else:
                if self._graphs[i] is None:
                    # first use of buffer set i: capture its forward (on the compute
                    # stream, after the upload it waits for), then replay it
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=self.s_comp):
                        backbone_forward(self.desc, self.packed, self.imgs[i],
                                         feats=self.feats[i], workspace=self.ws,
                                         stream=self.s_comp)
                    self._graphs[i] = g
                with torch.cuda.stream(self.s_comp):
                    self._graphs[i].replay()
            ev_comp[i].record(self.s_comp)
            self.s_out.wait_event(ev_comp[i])
            with torch.cuda.stream(self.s_out):
                for hf, f in zip(h_feats, self.feats[i]):
                    hf.copy_(f, non_blocking=True)
            ev_out[i].record(self.s_out)
            self._count += 1
        if end_event is not None:
            end_event.record(self.s_out)

    def synchronize(self):
        self.s_out.synchronize()
        self.s_comp.synchronize()
        self.s_in.synchronize()


# ----------------------------------------------------------------------------- status
def device_status(stream=None) -> int:
    """Synchronise and return (then clear) the first device-side error code."""
    return lib().hiera_get_device_status(_stream(stream))


def debug_gelu(x: torch.Tensor, stream=None) -> torch.Tensor:
    _need(x, "x")
    y = torch.empty_like(x)
    _check(lib().hiera_debug_gelu(_ptr(x), _ptr(y), x.numel(), _stream(stream)),
           "hiera_debug_gelu")
    return y


def timeout_probe(limit_us: int, stream=None):
    _check(lib().hiera_debug_timeout_probe(limit_us, _stream(stream)), "hiera_debug_timeout_probe")


def status_string(code: int) -> str:
    return lib().hiera_status_string(code).decode()


def kernel_name(kind: int) -> str:
    return lib().hiera_kernel_name(kind).decode()


# ----------------------------------------------------------------------------- options
OPT_FUSED_MLP = 0
OPT_PDL = 1
OPT_FUSED_ATTN = 2
OPT_GEMM224 = 3
GEMM224_EIGHT_WARPS, GEMM224_SIXTEEN_WARPS, GEMM224_PAIR = 0, 1, 2
OPT_SPLIT_BATCH = 4


def set_option(opt: int, value: int):
    _check(lib().hiera_set_option(opt, int(value)), "hiera_set_option")


def get_option(opt: int) -> int:
    return lib().hiera_get_option(opt)


class option:
    """Context manager: set a library option for the duration of a block of calls."""

    def __init__(self, opt: int, value: int):
        self.opt, self.value = opt, int(value)

    def __enter__(self):
        self._old = get_option(self.opt)
        set_option(self.opt, self.value)
        return self

    def __exit__(self, *exc):
        set_option(self.opt, self._old)
        return False


def fused_mlp(enabled: bool) -> option:
    """Run the block MLPs fused (True, the default) or as two GEMMs."""
    return option(OPT_FUSED_MLP, bool(enabled))


def fused_attention(enabled: bool) -> option:
    """Run the stage-0 blocks' attention half (norm1, qkv, windowed attention, proj,
    residual) as one kernel (True, the default) or as the separate kernels, which also write
    q, k, v and the attention output to the workspace."""
    return option(OPT_FUSED_ATTN, bool(enabled))


def gemm224(mode: int) -> option:
    """Kernel for the 224-column-tile Linear layers: GEMM224_EIGHT_WARPS (the default: one
    CTA per 128 x 224 tile, eight epilogue warps), GEMM224_SIXTEEN_WARPS (one CTA, sixteen
    epilogue warps) or GEMM224_PAIR (a CTA pair per 256 x 224 tile, tcgen05.mma.cta_group::2)."""
    return option(OPT_GEMM224, int(mode))


def split_batch(enabled: bool) -> option:
    """Run a backbone call's images as two concurrent half batches on two streams (True,
    the default, for B >= 2) or as one batch on the call's stream."""
    return option(OPT_SPLIT_BATCH, bool(enabled))


def pdl(enabled: bool) -> option:
    """Launch with programmatic dependent launch (True, the default) or plain launches."""
    return option(OPT_PDL, bool(enabled))


class LaunchProfile:
    """Marks every library launch with a CUDA event (see hiera_profile_begin).

    with LaunchProfile(capacity) as prof:  ... library calls on one stream ...
    prof.durations_ms() -> list of (kernel name, ms) once the work has completed.
    """

    def __init__(self, capacity: int = 512, stream=None):
        self.capacity = capacity
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(capacity)]
        for e in self.events:      # torch creates the CUDA event on first record
            e.record()
        torch.cuda.synchronize()
        self._handles = (ctypes.c_void_p * capacity)(*[e.cuda_event for e in self.events])
        self._kinds = (ctypes.c_int * capacity)()
        self.stream = stream
        self.count = 0

    def __enter__(self):
        _check(lib().hiera_profile_begin(self._handles, self.capacity, self._kinds),
               "hiera_profile_begin")
        return self

    def __exit__(self, *exc):
        self.count = lib().hiera_profile_end(_stream(self.stream))
        return False

    def durations_ms(self):
        n = min(self.count, self.capacity - 1)
        return [(kernel_name(self._kinds[i]), self.events[i].elapsed_time(self.events[i + 1]))
                for i in range(n)]
