"""Reader for routed-expert weights in the paired48 sparse storage of a
compressed-tensors checkpoint ("Sparse storage layout (paired48_sparse,
pair-bitmask v1)" of the Qwen3.5-397B-A17B-P48NVFP4-MoESQ model card).

Each routed-expert linear stores
    weight_sparse_packed   uint8 [out, K/4]    the 2 kept bytes of every 4, in K order
    weight_sparse_mask     uint8 [out, K/16]   4 bits per 4-byte chunk, exactly 2 set
    weight_scale           float8_e4m3 [out, K/32] block scales, linear layout
    weight_global_scale    float32             per-tensor global scale
    input_global_scale     float32             per-tensor activation global scale
and the quantization config carries "paired48_sparse": {"layout": "pair-bitmask",
"version": 1}.  The card gives no tensor names beyond these suffixes, so the caller
names each linear with a template (default: Hugging Face MoE names,
"{prefix}.experts.{e}.{proj}"), and it does not say whether a stored global is the
multiplier the dequantisation applies or its reciprocal.  The card does say the
checkpoints are in the compressed-tensors NVFP4 ("nvfp4-pack-quantized") form,
whose published convention stores the reciprocal, 6 * 448 / amax; the library works
with the multiplier, amax / (6 * 448).  The reader therefore decides from the
stored numbers (``global_convention="auto"``, the default) and refuses a reading
that the numbers contradict:

    read as a multiplier g, a block scale s dequantises to at most 6 * s * g, so the
    largest weight the stored tensor can hold is A_m = 6 * s_max * g; read as a
    reciprocal it is A_r = 6 * s_max / g.  A_m * A_r = (6 * s_max)**2, so exactly one
    of them is below 6 * s_max (2688 when a block reaches the E4M3 maximum 448) unless
    g == 1: a weight tensor whose largest element is thousands of times its own
    quantisation range does not exist, so that one is the reading.

An explicit ``global_convention`` ("multiplier" or "reciprocal") is checked the same
way and raises CheckpointError when the stored numbers say otherwise.  The input
global of a linear follows the convention of its weight global.

The safetensors container is parsed here directly (8-byte little-endian header
length, JSON header of name -> dtype, shape, data offsets; raw data after it); a
sharded checkpoint is found through its ``model.safetensors.index.json``.
Sparsity itself (exactly 2 bits per nibble) is checked on the device by the
repack and decode calls, which flag violations in their status word.
"""
from __future__ import annotations

import json
import mmap
import os
import struct

import numpy as np
import torch

MARKER = {"layout": "pair-bitmask", "version": 1}
SUFFIXES = ("weight_sparse_packed", "weight_sparse_mask", "weight_scale", "weight_global_scale",
            "input_global_scale")

_DTYPES = {"U8": (np.uint8, 1), "F8_E4M3": (np.uint8, 1), "F32": (np.float32, 4), "F16": (np.float16, 2),
           "BF16": (np.uint16, 2), "I32": (np.int32, 4), "I64": (np.int64, 8)}


class CheckpointError(ValueError):
    pass


class SafetensorsFile:
    """One .safetensors file, memory-mapped; tensors come out as numpy arrays (copies)."""

    def __init__(self, path: str):
        self.path = path
        with open(path, "rb") as f:
            head = f.read(8)
            if len(head) != 8:
                raise CheckpointError(f"{path}: truncated header length")
            (n,) = struct.unpack("<Q", head)
            if n > 100 * 1024 * 1024:
                raise CheckpointError(f"{path}: header of {n} bytes")
            try:
                self.header = json.loads(f.read(n).decode("utf-8"))
            except (UnicodeDecodeError, json.JSONDecodeError) as ex:
                raise CheckpointError(f"{path}: bad header ({ex})") from None
        self.data_start = 8 + n
        self.size = os.path.getsize(path)
        self.metadata = self.header.pop("__metadata__", {}) or {}

    def names(self):
        return list(self.header)

    def get(self, name: str) -> np.ndarray:
        if name not in self.header:
            raise KeyError(name)
        ent = self.header[name]
        dt = ent["dtype"]
        if dt not in _DTYPES:
            raise CheckpointError(f"{name}: dtype {dt} not supported")
        npdt, size = _DTYPES[dt]
        b0, b1 = ent["data_offsets"]
        shape = tuple(ent["shape"])
        count = int(np.prod(shape)) if shape else 1
        if b1 - b0 != count * size or self.data_start + b1 > self.size or b0 < 0 or b1 < b0:
            raise CheckpointError(f"{name}: data offsets {b0}..{b1} do not match {dt} {list(shape)}")
        with open(self.path, "rb") as f, mmap.mmap(f.fileno(), 0, access=mmap.ACCESS_READ) as m:
            buf = m[self.data_start + b0:self.data_start + b1]
        return np.frombuffer(buf, dtype=npdt).reshape(shape).copy()


class Checkpoint:
    """A checkpoint directory (one file, or shards with model.safetensors.index.json)."""

    def __init__(self, directory: str):
        self.directory = directory
        idx = os.path.join(directory, "model.safetensors.index.json")
        if os.path.exists(idx):
            wm = json.load(open(idx))["weight_map"]
            files = sorted(set(wm.values()))
            self._files = {f: SafetensorsFile(os.path.join(directory, f)) for f in files}
            self._where = {name: self._files[f] for name, f in wm.items()}
        else:
            files = sorted(f for f in os.listdir(directory) if f.endswith(".safetensors"))
            if not files:
                raise CheckpointError(f"{directory}: no .safetensors files")
            self._files = {f: SafetensorsFile(os.path.join(directory, f)) for f in files}
            self._where = {}
            for sf in self._files.values():
                for n in sf.names():
                    self._where[n] = sf
        cfg = os.path.join(directory, "config.json")
        self.config = json.load(open(cfg)) if os.path.exists(cfg) else {}

    def __contains__(self, name):
        return name in self._where

    def get(self, name: str) -> np.ndarray:
        if name not in self._where:
            raise CheckpointError(f"tensor {name} not in the checkpoint")
        return self._where[name].get(name)

    def check_marker(self):
        """The quantization config must declare paired48 sparse storage, pair-bitmask v1."""
        qc = self.config.get("quantization_config", {})
        mk = qc.get("paired48_sparse")
        if mk is None:
            raise CheckpointError("quantization_config has no paired48_sparse marker")
        if mk.get("layout") != MARKER["layout"] or int(mk.get("version", -1)) != MARKER["version"]:
            raise CheckpointError(f"unsupported paired48_sparse storage {mk}")


def _scalar(a: np.ndarray, name: str) -> np.float32:
    a = np.asarray(a, np.float32).reshape(-1)
    if a.size != 1:
        raise CheckpointError(f"{name}: expected one float32 value, got shape {list(a.shape)}")
    return a[0]


CONVENTIONS = ("auto", "multiplier", "reciprocal")


def stored_convention(g: np.float32, scale_codes: np.ndarray):
    """'multiplier' or 'reciprocal': the reading of a stored weight global under which
    the largest weight the tensor can hold (6 * largest block scale * multiplier) stays
    below 6 * largest block scale; None when the numbers cannot tell (g == 1, no
    nonzero block scale, or a global that is not finite and positive)."""
    s_max = float(torch.from_numpy(np.ascontiguousarray(scale_codes)).view(torch.float8_e4m3fn).float()
                  .nan_to_num(0.0).abs().max()) if scale_codes.size else 0.0
    g = float(g)
    if not (np.isfinite(g) and g > 0) or s_max == 0.0 or g == 1.0:
        return None
    a_mult, a_recip = 6.0 * s_max * g, 6.0 * s_max / g
    return "multiplier" if a_mult < a_recip else "reciprocal"


def read_linear(ckpt: Checkpoint, name: str, global_convention: str = "auto") -> dict:
    """One expert linear -> dict(packed [out,K/4] u8, mask [out,K/16] u8, scale [out,K/32]
    u8 (E4M3 codes), g (weight global multiplier, float32), g_in (activation global
    multiplier, float32), convention (how the file stored them))."""
    if global_convention not in CONVENTIONS:
        raise ValueError(f"global_convention is one of {CONVENTIONS}")
    packed = ckpt.get(f"{name}.weight_sparse_packed")
    mask = ckpt.get(f"{name}.weight_sparse_mask")
    scale = ckpt.get(f"{name}.weight_scale")
    if packed.ndim != 2 or mask.ndim != 2 or scale.ndim != 2:
        raise CheckpointError(f"{name}: storage tensors must be 2-D")
    out, k4 = packed.shape
    K = 4 * k4
    if mask.shape != (out, K // 16) or scale.shape != (out, K // 32) or K % 32:
        raise CheckpointError(f"{name}: shapes packed {packed.shape}, mask {mask.shape}, scale {scale.shape} "
                              f"do not describe one [out, K] paired-4:8 NVFP4 weight")
    g = _scalar(ckpt.get(f"{name}.weight_global_scale"), f"{name}.weight_global_scale")
    g_in = _scalar(ckpt.get(f"{name}.input_global_scale"), f"{name}.input_global_scale")
    seen = stored_convention(g, scale)
    conv = global_convention
    if conv == "auto":
        if seen is None:
            fmt = str(ckpt.config.get("quantization_config", {}).get("format", ""))
            if fmt != "nvfp4-pack-quantized":
                raise CheckpointError(f"{name}: cannot tell whether the stored global {float(g)!r} is a multiplier "
                                      f"or its reciprocal; pass global_convention")
            seen = "reciprocal"        # the compressed-tensors NVFP4 convention
        conv = seen
    elif seen is not None and seen != conv:
        raise CheckpointError(f"{name}: the stored global {float(g)!r} with block scales up to the stored maximum "
                              f"is a {seen}, not a {conv}")
    if conv == "reciprocal":
        g, g_in = np.float32(1) / g, np.float32(1) / g_in
    return dict(packed=packed, mask=mask, scale=scale, g=np.float32(g), g_in=np.float32(g_in), out=out, K=K,
                convention=conv)


def read_moe_experts(ckpt: Checkpoint, prefix: str, E: int, template: str = "{prefix}.experts.{e}.{proj}",
                     projs=("gate_proj", "up_proj", "down_proj"), global_convention: str = "auto",
                     check_marker: bool = True) -> dict:
    """All routed experts of one MoE layer, in the library's storage form.

    Returns dict(gate_up=dict(packed [E,2I,K/4], mask, scale, g_w [E,2] (gate, up)),
                 down=dict(packed [E,H,I/4], mask, scale, g_w [E,1]),
                 g_in_gate_up [E], g_in_down [E]) as host tensors; the fused gate_up
    stacks the gate rows above the up rows.  The activation global of gate_up is the
    one stored with gate_proj, and up_proj's must equal it (both quantise the same
    input).  Every linear of the layer must have stored its globals the same way."""
    if check_marker:
        ckpt.check_marker()
    gate, up, down = projs
    gu_p, gu_m, gu_s, gu_g, g_in_gu = [], [], [], [], []
    dn_p, dn_m, dn_s, dn_g, g_in_dn = [], [], [], [], []
    shapes = None
    first_conv = None
    for e in range(E):
        lg = read_linear(ckpt, template.format(prefix=prefix, e=e, proj=gate), global_convention)
        lu = read_linear(ckpt, template.format(prefix=prefix, e=e, proj=up), global_convention)
        ld = read_linear(ckpt, template.format(prefix=prefix, e=e, proj=down), global_convention)
        if lg["out"] != lu["out"] or lg["K"] != lu["K"] or ld["K"] != lg["out"] or ld["out"] != lg["K"]:
            raise CheckpointError(f"expert {e}: gate {lg['out']}x{lg['K']}, up {lu['out']}x{lu['K']}, "
                                  f"down {ld['out']}x{ld['K']} do not form one MLP")
        sh = (lg["out"], lg["K"])
        if shapes is None:
            shapes = sh
        elif sh != shapes:
            raise CheckpointError(f"expert {e}: shape {sh} differs from expert 0's {shapes}")
        convs = {lg["convention"], lu["convention"], ld["convention"]}
        if len(convs) > 1 or (e > 0 and convs != {first_conv}):
            raise CheckpointError(f"expert {e}: globals stored in mixed conventions {sorted(convs)}")
        first_conv = lg["convention"]
        if lg["g_in"] != lu["g_in"]:
            raise CheckpointError(f"expert {e}: gate and up input globals differ ({lg['g_in']} vs {lu['g_in']})")
        gu_p.append(np.concatenate([lg["packed"], lu["packed"]]))
        gu_m.append(np.concatenate([lg["mask"], lu["mask"]]))
        gu_s.append(np.concatenate([lg["scale"], lu["scale"]]))
        gu_g.append([lg["g"], lu["g"]])
        g_in_gu.append(lg["g_in"])
        dn_p.append(ld["packed"])
        dn_m.append(ld["mask"])
        dn_s.append(ld["scale"])
        dn_g.append([ld["g"]])
        g_in_dn.append(ld["g_in"])

    def pack(p, m, s, g):
        t = dict(packed=torch.from_numpy(np.stack(p)), mask=torch.from_numpy(np.stack(m)),
                 scale=torch.from_numpy(np.stack(s)), g_w=torch.from_numpy(np.asarray(g, np.float32)))
        E_, out, k4 = t["packed"].shape
        t.update(E=E_, out=out, K=4 * k4)
        return t

    return dict(gate_up=pack(gu_p, gu_m, gu_s, gu_g), down=pack(dn_p, dn_m, dn_s, dn_g),
                g_in_gate_up=torch.from_numpy(np.asarray(g_in_gu, np.float32)),
                g_in_down=torch.from_numpy(np.asarray(g_in_dn, np.float32)))


def to_device(storage: dict, device) -> dict:
    """Host storage dict (read_moe_experts) -> the same tensors on ``device``."""
    out = dict(storage)
    for k in ("packed", "mask", "scale", "g_w"):
        out[k] = storage[k].to(device).contiguous()
    return out


def load_moe_layer(directory: str, prefix: str, E: int, k: int, exact: bool = False, device="cuda",
                   **read_kw):
    """Read one MoE layer's routed experts and build the library's layer on ``device``
    (the load-time repack runs on the device).  ``exact``: keep the gate and up
    globals apart (GATE_UP_EXACT) instead of folding their ratio into the up scales."""
    from .layer import KIND_DOWN, KIND_GATE_UP_EXACT, KIND_GATE_UP_SPLIT, ExpertLinear, MoELayer

    st = read_moe_experts(Checkpoint(directory), prefix, E, **read_kw)
    gu = ExpertLinear.from_storage(to_device(st["gate_up"], device),
                                   KIND_GATE_UP_EXACT if exact else KIND_GATE_UP_SPLIT)
    dn = ExpertLinear.from_storage(to_device(st["down"], device), KIND_DOWN)
    return MoELayer(k, gu, dn, st["g_in_gate_up"].to(device), st["g_in_down"].to(device))
