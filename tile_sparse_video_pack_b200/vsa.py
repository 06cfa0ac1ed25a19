"""ctypes binding of libvsa (argument marshalling only).

Every step of the layer runs in the CUDA library; this module checks tensor
types, shapes and devices, and passes raw pointers and the current CUDA stream.
PyTorch is used only to allocate device memory and to name streams. If the
library is missing the import fails: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libvsa.so")

MAX_HEADS = 64
MAX_SEGMENTS = 8
TILE = 64

VSA_OK = 0
STATUS_NAMES = {0: "VSA_OK", 1: "VSA_ERR_INVALID_ARG", 2: "VSA_ERR_UNSUPPORTED", 3: "VSA_ERR_CUDA",
                4: "VSA_ERR_DEVICE_TIMEOUT", 5: "VSA_ERR_BAD_INDEX", 6: "VSA_ERR_NO_MEMORY"}
SCORE_MODES = {"meanpool_gate": 0, "tripool": 1}

# every entry point declared in include/vsa.h
EXPORTS = ("vsa_plan_create", "vsa_plan_destroy", "vsa_plan_query", "vsa_plan_get_stats", "vsa_k_from_sparsity",
           "vsa_tile_pack", "vsa_tile_score", "vsa_topk_select", "vsa_sparse_attn", "vsa_tile_unpack",
           "vsa_layer_forward", "vsa_plan_check", "vsa_status_string", "vsa_tile_score_static",
           "vsa_tile_pack_pool", "vsa_tile_score_pooled", "vsa_teacher_tiles", "vsa_index_overlap",
           "vsa_ref_score", "vsa_topk_select_ref", "vsa_sparse_attn_ref", "vsa_tile_pack_pool_fp8",
           "vsa_sparse_attn_fp8", "vsa_plan_set_wait_limit", "vsa_plan_set_test_hold", "vsa_tile_pool",
           "vsa_sparse_attn_direct")


class VsaDesc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("T", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32),
        ("n_segments", ctypes.c_int32), ("seg_len", ctypes.c_int32 * MAX_SEGMENTS),
        ("tile_shape", (ctypes.c_int32 * 3) * MAX_HEADS),
        ("k_per_head", ctypes.c_int32 * MAX_HEADS),
        ("score_mode", ctypes.c_int32), ("proj_dim", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
        ("seg_ref", ctypes.c_int32 * MAX_SEGMENTS), ("k_ref_per_head", ctypes.c_int32 * MAX_HEADS),
    ]


class VsaPlanInfo(ctypes.Structure):
    _fields_ = [
        ("n_tokens", ctypes.c_int64), ("n_prefix_tiles", ctypes.c_int32), ("nt_max", ctypes.c_int32),
        ("ntv_max", ctypes.c_int32), ("ntv", ctypes.c_int32 * MAX_HEADS), ("k_max", ctypes.c_int32),
        ("packed_elems", ctypes.c_int64), ("score_elems", ctypes.c_int64), ("index_elems", ctypes.c_int64),
        ("workspace_bytes", ctypes.c_int64), ("lse_elems", ctypes.c_int64), ("attn_work_items", ctypes.c_int64),
        ("n_ref_tiles", ctypes.c_int32), ("k_ref_max", ctypes.c_int32),
        ("ref_score_elems", ctypes.c_int64), ("ref_index_elems", ctypes.c_int64),
        ("tile_scale_elems", ctypes.c_int64), ("direct_attn", ctypes.c_int32), ("reserved0", ctypes.c_int32),
    ]


class VsaPlanStats(ctypes.Structure):
    _fields_ = [
        ("calls_pack", ctypes.c_int64), ("calls_score", ctypes.c_int64), ("calls_select", ctypes.c_int64),
        ("calls_attn", ctypes.c_int64), ("calls_unpack", ctypes.c_int64), ("errors", ctypes.c_int64),
        ("computed_pairs", ctypes.c_int64), ("dense_pairs", ctypes.c_int64),
    ]


class VsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


_lib = None


def library() -> ctypes.CDLL:
    """The loaded libvsa (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libvsa.so not built ({LIB_PATH}); run python -m tile_sparse_video_pack_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    sig = {
        "vsa_plan_create": (I32, [ctypes.POINTER(VsaDesc), ctypes.POINTER(P)]),
        "vsa_plan_destroy": (I32, [P]),
        "vsa_plan_query": (I32, [P, ctypes.POINTER(VsaPlanInfo)]),
        "vsa_plan_get_stats": (I32, [P, ctypes.POINTER(VsaPlanStats)]),
        "vsa_k_from_sparsity": (I32, [D, I32]),
        "vsa_tile_pack": (I32, [P, P, P, P, P, P, P, P]),
        "vsa_tile_score": (I32, [P, P, P, P, P, P, P, P]),
        "vsa_topk_select": (I32, [P, P, P, P, P]),
        "vsa_sparse_attn": (I32, [P, P, P, P, P, P, P, P, P]),
        "vsa_tile_unpack": (I32, [P, P, P, P]),
        "vsa_layer_forward": (I32, [P] + [P] * 15),
        "vsa_plan_check": (I32, [P]),
        "vsa_status_string": (ctypes.c_char_p, [I32]),
        "vsa_tile_score_static": (I32, [P, P, P, P, P, P, P]),
        "vsa_tile_pack_pool": (I32, [P] * 9),
        "vsa_tile_score_pooled": (I32, [P] * 6),
        "vsa_teacher_tiles": (I32, [P] * 6),
        "vsa_index_overlap": (I32, [P] * 6),
        "vsa_ref_score": (I32, [P] * 6),
        "vsa_topk_select_ref": (I32, [P] * 4),
        "vsa_sparse_attn_ref": (I32, [P] * 10),
        "vsa_tile_pack_pool_fp8": (I32, [P] * 13),
        "vsa_sparse_attn_fp8": (I32, [P] * 11),
        "vsa_plan_set_wait_limit": (I32, [P, ctypes.c_uint64]),
        "vsa_plan_set_test_hold": (I32, [P, I32]),
        "vsa_tile_pool": (I32, [P] * 5),
        "vsa_sparse_attn_direct": (I32, [P] * 9),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    _lib = lib
    return lib


def k_from_sparsity(sparsity: float, n_tiles: int) -> int:
    return int(library().vsa_k_from_sparsity(float(sparsity), int(n_tiles)))


def _check(status: int, where: str):
    if status != VSA_OK:
        raise VsaError(status, where)


def make_desc(batch, heads, head_dim, T, H, W, segments, tile_shapes, k_per_head, score_mode="meanpool_gate",
              proj_dim=None, softmax_scale=0.0, seg_ref=(), k_ref_per_head=()) -> VsaDesc:
    d = VsaDesc()
    d.batch, d.heads, d.head_dim = batch, heads, head_dim
    d.T, d.H, d.W = T, H, W
    if len(segments) > MAX_SEGMENTS or heads > MAX_HEADS or len(tile_shapes) != heads or len(k_per_head) != heads:
        raise ValueError("descriptor does not fit vsa_desc")
    d.n_segments = len(segments)
    for i, s in enumerate(segments):
        d.seg_len[i] = s
    for h, shp in enumerate(tile_shapes):
        for a in range(3):
            d.tile_shape[h][a] = shp[a]
    for h, k in enumerate(k_per_head):
        d.k_per_head[h] = k
    d.score_mode = SCORE_MODES[score_mode] if isinstance(score_mode, str) else int(score_mode)
    d.proj_dim = head_dim if proj_dim is None else proj_dim
    d.softmax_scale = softmax_scale
    for i, f in enumerate(seg_ref):
        d.seg_ref[i] = int(f)
    for h, k in enumerate(k_ref_per_head):
        d.k_ref_per_head[h] = k
    return d


def _ptr(t, dtype, name, min_numel=0):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        # the library launches on the current device, which must also be the plan's
        raise ValueError(f"{name} is on {t.device}, but cuda:{torch.cuda.current_device()} is the current device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements, needs {min_numel}")
    return ctypes.c_void_p(t.data_ptr())


def _karray(k_per_head, heads):
    """A host int32 array of the per-call k of each head (None -> NULL: the plan's own k)."""
    if k_per_head is None:
        return None
    ks = [int(x) for x in k_per_head]
    if len(ks) != heads:
        raise ValueError(f"k_per_head has {len(ks)} entries, the plan {heads} heads")
    return (ctypes.c_int32 * heads)(*ks)


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Plan:
    """A vsa_plan: one layer's tiling tables and attention work list on the current device."""

    def __init__(self, desc: VsaDesc):
        lib = library()
        self.desc = desc
        h = ctypes.c_void_p()
        _check(lib.vsa_plan_create(ctypes.byref(desc), ctypes.byref(h)), "vsa_plan_create")
        self._h = h
        inf = VsaPlanInfo()
        _check(lib.vsa_plan_query(h, ctypes.byref(inf)), "vsa_plan_query")
        self.info = inf

    @classmethod
    def from_config(cls, cfg, sparsity: float, k_per_head=None):
        """Plan for a :class:`vsa_synth.configs.LayerConfig` at one sparsity level."""
        ks = k_per_head
        if ks is None:
            ks = []
            for (pt, ph, pw) in cfg.tile_shapes:
                n = -(-cfg.T // pt) * -(-cfg.H // ph) * -(-cfg.W // pw)
                ks.append(k_from_sparsity(sparsity, n))
        seg_ref = tuple(getattr(cfg, "seg_ref", ()))
        k_ref = [int(cfg.k_ref)] * cfg.heads if any(seg_ref) else []
        return cls(make_desc(cfg.batch, cfg.heads, cfg.head_dim, cfg.T, cfg.H, cfg.W, cfg.segments,
                             cfg.tile_shapes, ks, cfg.score_mode, cfg.proj_dim, seg_ref=seg_ref,
                             k_ref_per_head=k_ref))

    def close(self):
        if getattr(self, "_h", None):
            library().vsa_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---- shapes ----------------------------------------------------------------
    @property
    def k_per_head(self):
        return [self.desc.k_per_head[h] for h in range(self.desc.heads)]

    def shapes(self):
        d, i = self.desc, self.info
        return {
            "tokens": (d.batch, i.n_tokens, d.heads, d.head_dim),
            "packed": (d.batch, d.heads, i.nt_max, TILE, d.head_dim),
            "scores": (d.batch, d.heads, i.ntv_max, i.ntv_max),
            "idx": (d.batch, d.heads, i.ntv_max, i.k_max),
            "lse": (d.batch, d.heads, i.nt_max, TILE),
            "workspace": (i.workspace_bytes,),
            "scores_ref": (d.batch, d.heads, i.ntv_max, i.n_ref_tiles),
            "idx_ref": (d.batch, d.heads, i.ntv_max, i.k_ref_max),
        }

    def allocate(self, device=None, with_lse=False, packed=True):
        """Device buffers for every intermediate of the layer (torch is only the allocator).

        packed=False leaves out the packed tiles (qp, kp, vp, op: None), which a plan with
        info.direct_attn does not need."""
        import torch
        dev = torch.device("cuda") if device is None else torch.device(device)
        s = self.shapes()
        pk = (lambda: torch.empty(s["packed"], dtype=torch.bfloat16, device=dev)) if packed else (lambda: None)
        bufs = {
            "qp": pk(),
            "kp": pk(),
            "vp": pk(),
            "op": pk(),
            "scores": torch.empty(s["scores"], dtype=torch.float32, device=dev),
            "idx": torch.empty(s["idx"], dtype=torch.int32, device=dev),
            "workspace": torch.empty(s["workspace"], dtype=torch.uint8, device=dev),
            "lse": torch.empty(s["lse"], dtype=torch.float32, device=dev) if with_lse else None,
        }
        if self.info.n_ref_tiles:
            bufs["scores_ref"] = torch.empty(s["scores_ref"], dtype=torch.float32, device=dev)
            bufs["idx_ref"] = torch.empty(s["idx_ref"], dtype=torch.int32, device=dev)
        return bufs

    # ---- the five calls (same names as the C ABI) ------------------------------
    def tile_pack(self, q, k, v, qp, kp, vp, stream=None):
        import torch
        n_tok = self.desc.batch * self.info.n_tokens * self.desc.heads * self.desc.head_dim
        bf = torch.bfloat16
        args = [_ptr(x, bf, nm, n_tok) for x, nm in ((q, "q"), (k, "k"), (v, "v"))]
        outs = [_ptr(x, bf, nm, self.info.packed_elems) if src is not None else None
                for x, nm, src in ((qp, "qp", q), (kp, "kp", k), (vp, "vp", v))]
        _check(library().vsa_tile_pack(self._h, *args, *outs, _stream(stream)), "vsa_tile_pack")

    def tile_score(self, qp, kp, proj_q, proj_k, scores, workspace, stream=None):
        import torch
        pe = self.info.packed_elems
        _check(library().vsa_tile_score(
            self._h, _ptr(qp, torch.bfloat16, "qp", pe), _ptr(kp, torch.bfloat16, "kp", pe),
            _ptr(proj_q, torch.float32, "proj_q"), _ptr(proj_k, torch.float32, "proj_k"),
            _ptr(scores, torch.float32, "scores", self.info.score_elems),
            _ptr(workspace, torch.uint8, "workspace", self.info.workspace_bytes), _stream(stream)),
            "vsa_tile_score")

    def tile_pool(self, q, k, workspace, stream=None):
        """Pooling of the score stage straight from token-major q, k (plans with info.direct_attn)."""
        import torch
        n_tok = self.desc.batch * self.info.n_tokens * self.desc.heads * self.desc.head_dim
        bf = torch.bfloat16
        _check(library().vsa_tile_pool(
            self._h, _ptr(q, bf, "q", n_tok), _ptr(k, bf, "k", n_tok),
            _ptr(workspace, torch.uint8, "workspace", self.info.workspace_bytes), _stream(stream)),
            "vsa_tile_pool")

    def sparse_attn_direct(self, q, k, v, idx, o, lse=None, stream=None, k_per_head=None):
        """Attention from token-major q, k, v into token-major o (plans with info.direct_attn)."""
        import torch
        n_tok = self.desc.batch * self.info.n_tokens * self.desc.heads * self.desc.head_dim
        bf = torch.bfloat16
        _check(library().vsa_sparse_attn_direct(
            self._h, _ptr(q, bf, "q", n_tok), _ptr(k, bf, "k", n_tok), _ptr(v, bf, "v", n_tok),
            _ptr(idx, torch.int32, "idx", self.info.index_elems), _karray(k_per_head, self.desc.heads),
            _ptr(o, bf, "o", n_tok), _ptr(lse, torch.float32, "lse", self.info.lse_elems), _stream(stream)),
            "vsa_sparse_attn_direct")

    def tile_pack_pool(self, q, k, v, qp, kp, vp, workspace, stream=None):
        """tile_pack fused with the pooling of tile_score; follow with tile_score_pooled."""
        import torch
        n_tok = self.desc.batch * self.info.n_tokens * self.desc.heads * self.desc.head_dim
        pe, bf = self.info.packed_elems, torch.bfloat16
        _check(library().vsa_tile_pack_pool(
            self._h, _ptr(q, bf, "q", n_tok), _ptr(k, bf, "k", n_tok), _ptr(v, bf, "v", n_tok),
            _ptr(qp, bf, "qp", pe), _ptr(kp, bf, "kp", pe), _ptr(vp, bf, "vp", pe),
            _ptr(workspace, torch.uint8, "workspace", self.info.workspace_bytes), _stream(stream)),
            "vsa_tile_pack_pool")

    def tile_pack_pool_fp8(self, q, k, v, qp, kp, vp, qp8, kp8, q_scale, k_scale, workspace, stream=None):
        """tile_pack_pool plus e4m3 copies of Q and K with one fp32 scale per tile (head_dim 128)."""
        import torch
        n_tok = self.desc.batch * self.info.n_tokens * self.desc.heads * self.desc.head_dim
        pe, bf, u8, f32 = self.info.packed_elems, torch.bfloat16, torch.uint8, torch.float32
        ns = self.info.tile_scale_elems
        _check(library().vsa_tile_pack_pool_fp8(
            self._h, _ptr(q, bf, "q", n_tok), _ptr(k, bf, "k", n_tok), _ptr(v, bf, "v", n_tok),
            _ptr(qp, bf, "qp", pe), _ptr(kp, bf, "kp", pe), _ptr(vp, bf, "vp", pe),
            _ptr(qp8, u8, "qp8", pe), _ptr(kp8, u8, "kp8", pe), _ptr(q_scale, f32, "q_scale", ns),
            _ptr(k_scale, f32, "k_scale", ns),
            _ptr(workspace, u8, "workspace", self.info.workspace_bytes), _stream(stream)), "vsa_tile_pack_pool_fp8")

    def sparse_attn_fp8(self, qp8, kp8, q_scale, k_scale, vp, idx, op, lse=None, stream=None, k_per_head=None):
        """sparse_attn with Q K^T from the e4m3 tiles and their per-tile scales."""
        import torch
        pe, u8, f32, bf = self.info.packed_elems, torch.uint8, torch.float32, torch.bfloat16
        ns = self.info.tile_scale_elems
        _check(library().vsa_sparse_attn_fp8(
            self._h, _ptr(qp8, u8, "qp8", pe), _ptr(kp8, u8, "kp8", pe), _ptr(q_scale, f32, "q_scale", ns),
            _ptr(k_scale, f32, "k_scale", ns), _ptr(vp, bf, "vp", pe),
            _ptr(idx, torch.int32, "idx", self.info.index_elems), _karray(k_per_head, self.desc.heads),
            _ptr(op, bf, "op", pe),
            _ptr(lse, f32, "lse", self.info.lse_elems), _stream(stream)), "vsa_sparse_attn_fp8")

    def allocate_fp8(self, device=None):
        """The e4m3 Q, K tiles and their per-tile scales."""
        import torch
        dev = torch.device("cuda") if device is None else torch.device(device)
        pe, ns = self.info.packed_elems, self.info.tile_scale_elems
        return {"qp8": torch.empty(pe, dtype=torch.uint8, device=dev),
                "kp8": torch.empty(pe, dtype=torch.uint8, device=dev),
                "q_scale": torch.empty(ns, dtype=torch.float32, device=dev),
                "k_scale": torch.empty(ns, dtype=torch.float32, device=dev)}

    def tile_score_pooled(self, proj_q, proj_k, scores, workspace, stream=None):
        """Projection and scores from the descriptors tile_pack_pool left in the workspace."""
        import torch
        _check(library().vsa_tile_score_pooled(
            self._h, _ptr(proj_q, torch.float32, "proj_q"), _ptr(proj_k, torch.float32, "proj_k"),
            _ptr(scores, torch.float32, "scores", self.info.score_elems),
            _ptr(workspace, torch.uint8, "workspace", self.info.workspace_bytes), _stream(stream)),
            "vsa_tile_score_pooled")

    def teacher_tiles(self, qp, kp, lse, teacher, stream=None):
        """Max-pooled full-attention weights per video tile pair; lse from a dense sparse_attn."""
        import torch
        pe = self.info.packed_elems
        _check(library().vsa_teacher_tiles(
            self._h, _ptr(qp, torch.bfloat16, "qp", pe), _ptr(kp, torch.bfloat16, "kp", pe),
            _ptr(lse, torch.float32, "lse", self.info.lse_elems),
            _ptr(teacher, torch.float32, "teacher", self.info.score_elems), _stream(stream)), "vsa_teacher_tiles")

    def index_overlap(self, idx_a, idx_b, counts, stream=None, k_per_head=None):
        """Shared indices per row of two ascending top-k tables."""
        import torch
        n = self.desc.batch * self.desc.heads * self.info.ntv_max
        _check(library().vsa_index_overlap(
            self._h, _ptr(idx_a, torch.int32, "idx_a", self.info.index_elems),
            _ptr(idx_b, torch.int32, "idx_b", self.info.index_elems), _karray(k_per_head, self.desc.heads),
            _ptr(counts, torch.int32, "counts", n), _stream(stream)), "vsa_index_overlap")

    def tile_score_static(self, qp, kp, proj_q, proj_k, scores, stream=None):
        """tile_score with the library's fixed 32 MiB device scratch instead of a workspace.

        For callers that may not allocate device memory while the layer runs.
        Its first call on a device looks up the scratch address: make it before
        any stream capture. Calls that overlap on the GPU share the scratch and race.
        """
        import torch
        pe = self.info.packed_elems
        _check(library().vsa_tile_score_static(
            self._h, _ptr(qp, torch.bfloat16, "qp", pe), _ptr(kp, torch.bfloat16, "kp", pe),
            _ptr(proj_q, torch.float32, "proj_q"), _ptr(proj_k, torch.float32, "proj_k"),
            _ptr(scores, torch.float32, "scores", self.info.score_elems), _stream(stream)),
            "vsa_tile_score_static")

    def topk_select(self, scores, idx, stream=None, k_per_head=None):
        """k_per_head: this call's kept tiles per head (None: the plan's)."""
        import torch
        _check(library().vsa_topk_select(
            self._h, _ptr(scores, torch.float32, "scores", self.info.score_elems),
            _karray(k_per_head, self.desc.heads),
            _ptr(idx, torch.int32, "idx", self.info.index_elems), _stream(stream)), "vsa_topk_select")

    def sparse_attn(self, qp, kp, vp, idx, op, lse=None, stream=None, k_per_head=None):
        """k_per_head: this call's kept tiles per head (None: the plan's); as given to topk_select."""
        import torch
        pe, bf = self.info.packed_elems, torch.bfloat16
        _check(library().vsa_sparse_attn(
            self._h, _ptr(qp, bf, "qp", pe), _ptr(kp, bf, "kp", pe), _ptr(vp, bf, "vp", pe),
            _ptr(idx, torch.int32, "idx", self.info.index_elems), _karray(k_per_head, self.desc.heads),
            _ptr(op, bf, "op", pe),
            _ptr(lse, torch.float32, "lse", self.info.lse_elems), _stream(stream)), "vsa_sparse_attn")

    def ref_score(self, kp, proj_k, scores_ref, workspace, stream=None):
        """Scores of the reference tiles (R2VA budgets); after tile_score(_pooled) on the same workspace."""
        import torch
        _check(library().vsa_ref_score(
            self._h, _ptr(kp, torch.bfloat16, "kp", self.info.packed_elems), _ptr(proj_k, torch.float32, "proj_k"),
            _ptr(scores_ref, torch.float32, "scores_ref", self.info.ref_score_elems),
            _ptr(workspace, torch.uint8, "workspace", self.info.workspace_bytes), _stream(stream)), "vsa_ref_score")

    def topk_select_ref(self, scores_ref, idx_ref, stream=None):
        import torch
        _check(library().vsa_topk_select_ref(
            self._h, _ptr(scores_ref, torch.float32, "scores_ref", self.info.ref_score_elems),
            _ptr(idx_ref, torch.int32, "idx_ref", self.info.ref_index_elems), _stream(stream)),
            "vsa_topk_select_ref")

    def sparse_attn_ref(self, qp, kp, vp, idx, idx_ref, op, lse=None, stream=None, k_per_head=None):
        import torch
        pe, bf = self.info.packed_elems, torch.bfloat16
        _check(library().vsa_sparse_attn_ref(
            self._h, _ptr(qp, bf, "qp", pe), _ptr(kp, bf, "kp", pe), _ptr(vp, bf, "vp", pe),
            _ptr(idx, torch.int32, "idx", self.info.index_elems),
            _ptr(idx_ref, torch.int32, "idx_ref", self.info.ref_index_elems), _karray(k_per_head, self.desc.heads),
            _ptr(op, bf, "op", pe),
            _ptr(lse, torch.float32, "lse", self.info.lse_elems), _stream(stream)), "vsa_sparse_attn_ref")

    def tile_unpack(self, op, o, stream=None):
        import torch
        n_tok = self.desc.batch * self.info.n_tokens * self.desc.heads * self.desc.head_dim
        _check(library().vsa_tile_unpack(
            self._h, _ptr(op, torch.bfloat16, "op", self.info.packed_elems),
            _ptr(o, torch.bfloat16, "o", n_tok), _stream(stream)), "vsa_tile_unpack")

    def layer_forward(self, q, k, v, proj_q, proj_k, bufs, o, stream=None):
        """The layer's calls in one C-ABI call (vsa_layer_forward; the direct path when info.direct_attn)."""
        import torch
        pe, bf = self.info.packed_elems, torch.bfloat16
        n_tok = self.desc.batch * self.info.n_tokens * self.desc.heads * self.desc.head_dim
        _check(library().vsa_layer_forward(
            self._h, _ptr(q, bf, "q", n_tok), _ptr(k, bf, "k", n_tok), _ptr(v, bf, "v", n_tok),
            _ptr(proj_q, torch.float32, "proj_q"), _ptr(proj_k, torch.float32, "proj_k"),
            _ptr(bufs.get("qp"), bf, "qp", pe), _ptr(bufs.get("kp"), bf, "kp", pe), _ptr(bufs.get("vp"), bf, "vp", pe),
            _ptr(bufs["scores"], torch.float32, "scores", self.info.score_elems),
            _ptr(bufs["idx"], torch.int32, "idx", self.info.index_elems), _ptr(bufs.get("op"), bf, "op", pe),
            _ptr(bufs.get("lse"), torch.float32, "lse", self.info.lse_elems),
            _ptr(bufs["workspace"], torch.uint8, "workspace", self.info.workspace_bytes),
            _ptr(o, bf, "o", n_tok), _stream(stream)), "vsa_layer_forward")

    def set_wait_limit(self, limit_ns: int = 0):
        """Bound of every device-side wait of the plan's tcgen05 kernels (0: the two-second default)."""
        _check(library().vsa_plan_set_wait_limit(self._h, int(limit_ns)), "vsa_plan_set_wait_limit")

    def set_test_hold(self, on: bool):
        """Test hook: attention's softmax waits for a release nothing gives, until the wait limit."""
        _check(library().vsa_plan_set_test_hold(self._h, 1 if on else 0), "vsa_plan_set_test_hold")

    def check(self):
        """Synchronise and raise if a kernel latched a device-side error."""
        _check(library().vsa_plan_check(self._h), "vsa_plan_check")

    def stats(self) -> dict:
        st = VsaPlanStats()
        _check(library().vsa_plan_get_stats(self._h, ctypes.byref(st)), "vsa_plan_get_stats")
        return {name: getattr(st, name) for name, _ in VsaPlanStats._fields_}
