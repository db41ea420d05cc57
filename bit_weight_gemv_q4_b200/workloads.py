"""Tensor shapes of the single-user decode workloads.

A dense ~27B hybrid model with 64 layers, 16 of them gated attention and 48
Gated DeltaNet (wiselychen guide "Qwen3.8-27B measured ...", section "Before
deploying: weights, KV cache, memory bandwidth"), hidden size 5120, FFN width
17408, grouped k/v width 1024, vocabulary 248320; the attention projections
and the output head are raised to 8 bits while the rest stays at 4 bits
(bs178.com llamAmpere post, "Why it is this fast", part two).  The pages do not
give the DeltaNet projection shapes; every mixer here uses the q/k/v/o shapes
of the attention layers, and layer i is an attention layer when i % 4 == 3.
The draft head's vocabulary map keeps 65536 of the 248320 tokens (bs178.com
post, part four).

Algorithmic weight bytes per tensor: N*K/2 + 2*N*K/32 (q4) and
N*K + 2*N*K/32 (q8): the integer codes plus one fp16 scale per group of 32.
NVFP4 tensors (bits = NVFP4) hold N*K/2 code bytes plus one E4M3 byte per 16
values, N*K/16: the same 4.5 bits per weight as q4.
"""
from __future__ import annotations

from dataclasses import dataclass

HIDDEN = 5120
FFN = 17408
KV = 1024
VOCAB = 248320
DRAFT_VOCAB = 65536
N_LAYERS = 64
NVFP4 = 16  # the format id of NVFP4 tensors (the library's Q4_FMT_NVFP4)


def weight_bytes(bits: int, N: int, K: int) -> int:
    """Algorithmic bytes of one N x K tensor (codes + scales)."""
    if bits == NVFP4:
        return N * K // 2 + N * (K // 16)
    codes = N * K // 2 if bits == 4 else N * K
    return codes + 2 * N * (K // 32)


@dataclass(frozen=True)
class Tensor:
    name: str
    bits: int
    N: int
    K: int
    tensor_id: int  # selects the generator streams

    @property
    def bytes(self) -> int:
        return weight_bytes(self.bits, self.N, self.K)


def is_attention_layer(layer: int) -> bool:
    return layer % 4 == 3


def _layer_tensors(layer: int, mixer_bits: int, fused: bool) -> list[Tensor]:
    base = 16 + 16 * layer
    if fused:
        return [
            Tensor(f"L{layer}.qkv", mixer_bits, HIDDEN + 2 * KV, HIDDEN, base + 7),
            Tensor(f"L{layer}.o", mixer_bits, HIDDEN, HIDDEN, base + 3),
            Tensor(f"L{layer}.gate_up", 4, 2 * FFN, HIDDEN, base + 8),
            Tensor(f"L{layer}.down", 4, HIDDEN, FFN, base + 6),
        ]
    return [
        Tensor(f"L{layer}.q", mixer_bits, HIDDEN, HIDDEN, base + 0),
        Tensor(f"L{layer}.k", mixer_bits, KV, HIDDEN, base + 1),
        Tensor(f"L{layer}.v", mixer_bits, KV, HIDDEN, base + 2),
        Tensor(f"L{layer}.o", mixer_bits, HIDDEN, HIDDEN, base + 3),
        Tensor(f"L{layer}.gate", 4, FFN, HIDDEN, base + 4),
        Tensor(f"L{layer}.up", 4, FFN, HIDDEN, base + 5),
        Tensor(f"L{layer}.down", 4, HIDDEN, FFN, base + 6),
    ]


def single_q4() -> list[Tensor]:
    """One q4 4096 x 4096 product (M = 1)."""
    return [Tensor("w4096", 4, 4096, 4096, 1)]


def layer_q4() -> list[Tensor]:
    """One 27B-shaped layer, every projection q4 (used at M = 1 and M = 4)."""
    return _layer_tensors(0, 4, fused=False)


def draft_heads() -> list[Tensor]:
    """The q8 vocabulary projection, mapped (65536 rows) and full (248320 rows)."""
    return [Tensor("head.mapped", 8, DRAFT_VOCAB, HIDDEN, 1022), Tensor("head.full", 8, VOCAB, HIDDEN, 1023)]


def decode_stream(fused: bool = True) -> list[Tensor]:
    """The 64-layer weight stream of one decode step plus the q8 output head,
    in execution order.  fused=True concatenates the products that share an
    input (q|k|v and gate|up), 4 products per layer; fused=False lists all 7."""
    out: list[Tensor] = []
    for layer in range(N_LAYERS):
        out += _layer_tensors(layer, 8 if is_attention_layer(layer) else 4, fused)
    out.append(Tensor("head", 8, VOCAB, HIDDEN, 1023))
    return out


def as_nvfp4(tensors: list[Tensor]) -> list[Tensor]:
    """The same list with every q4 tensor in NVFP4 instead (q8 tensors kept):
    the same shapes and the same weight bytes."""
    return [Tensor(t.name, NVFP4, t.N, t.K, t.tensor_id) if t.bits == 4 else t for t in tensors]


def total_bytes(tensors: list[Tensor]) -> int:
    return sum(t.bytes for t in tensors)


def distinct_k(tensors: list[Tensor]) -> list[int]:
    return sorted({t.K for t in tensors})


def activation_stream_id(K: int) -> int:
    """Generator stream of the activations that feed every product with this K."""
    return K


class DeviceStream:
    """A list of products generated, packed and captured on the current CUDA
    device: the weights of every tensor (generated on the device from the
    seeded generator, then repacked by the library's device packer), one
    activation block per distinct K, one output per tensor, and the captured
    layer stack.  The oracle regenerates any row on the host from the same
    (seed, tensor id)."""

    def __init__(self, tensors: list[Tensor], M: int, seed: int = 0, flags: int = 0):
        import torch

        import bit_weight_gemv_q4_b200 as q4

        from . import synth

        self.tensors = list(tensors)
        self.M = M
        self.seed = seed
        dev = torch.device("cuda")
        max_canon = max((t.N * (t.K if t.bits == 8 else t.K // 2) for t in self.tensors), default=0)
        max_scales = max((t.N * (t.K // 16 if t.bits == NVFP4 else t.K // 32 * 2) for t in self.tensors), default=0)
        canon = torch.empty(max(max_canon, 16), dtype=torch.uint8, device=dev)
        scales = torch.empty(max(max_scales, 16), dtype=torch.uint8, device=dev)
        self.packed = []
        for t in self.tensors:
            nq = t.N * (t.K if t.bits == 8 else t.K // 2)
            if t.bits == NVFP4:  # codes from the q4 code stream, E4M3 scales from the scale stream
                ns = t.N * (t.K // 16)
                synth.weights_device(4, seed, synth.weight_stream(t.tensor_id), t.K, 0, t.N, canon[:nq])
                synth.e4m3_scales_device(seed, synth.scale_stream(t.tensor_id), t.K, 0, t.N, scales[:ns])
                p = torch.empty(q4.q4_nvfp4_packed_bytes(t.N, t.K), dtype=torch.uint8, device=dev)
                q4.q4_pack_nvfp4_device(canon[:nq], scales[:ns], synth.NVFP4_TENSOR_SCALE, t.N, t.K, p)
            else:
                ns = t.N * (t.K // 32)
                s16 = scales[: 2 * ns].view(torch.int16)
                synth.weights_device(t.bits, seed, synth.weight_stream(t.tensor_id), t.K, 0, t.N, canon[:nq])
                synth.scales_device(seed, synth.scale_stream(t.tensor_id), t.K, 0, t.N, s16)
                p = torch.empty(q4.q4_packed_bytes(t.bits, t.N, t.K), dtype=torch.uint8, device=dev)
                q4.q4_pack_weights_device(t.bits, canon[:nq], s16, t.N, t.K, p)
            self.packed.append(p)
        del canon, scales
        self.x = {}
        for K in distinct_k(self.tensors):
            xb = torch.empty(M * K, dtype=torch.int16, device=dev)
            synth.activations_device(seed, synth.act_stream(activation_stream_id(K)), M, K, xb)
            self.x[K] = xb
        self.y = [torch.empty(M * t.N, dtype=torch.float32, device=dev) for t in self.tensors]
        torch.cuda.synchronize()
        self.stack = self.make_stack(flags)

    def make_stack(self, flags: int = 0):
        """Another layer stack over the same device buffers (e.g. another mode)."""
        import bit_weight_gemv_q4_b200 as q4

        entries = [(t.bits, t.N, t.K, p, self.x[t.K], y) for t, p, y in zip(self.tensors, self.packed, self.y)]
        return q4.layer_stack_create(entries, self.M, flags)

    @property
    def weight_bytes(self) -> int:
        return total_bytes(self.tensors)

    def run(self, stream=None) -> None:
        import bit_weight_gemv_q4_b200 as q4

        q4.layer_stack_run(self.stack, stream)

    def check(self, stream=None) -> None:
        import bit_weight_gemv_q4_b200 as q4

        q4.layer_stack_check(self.stack, stream)

    def close(self) -> None:
        self.stack.close()
        self.packed.clear()
        self.y.clear()
        self.x.clear()


# ----------------------------------------------------------------------------
# The dependent decode chain: the same products, with the steps between them
# (residual + RMSNorm before q|k|v and gate|up, SwiGLU before down, a final
# norm before the head).  The attention / DeltaNet mixer is not computed: its
# output (the o projection's input) is an input of the step.
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class ChainShape:
    layers: int = N_LAYERS
    hidden: int = HIDDEN
    ffn: int = FFN
    kv: int = KV
    vocab: int = VOCAB


CHAIN_INPUT_BASE = 1 << 24  # generator streams of the chain's own inputs (beyond every K used as a stream id)


def chain_tensors(shape: ChainShape) -> list[Tensor]:
    """The chain's products in execution order (the default shape gives
    exactly decode_stream(fused=True))."""
    out: list[Tensor] = []
    H, F, KVW = shape.hidden, shape.ffn, shape.kv
    for layer in range(shape.layers):
        mb = 8 if is_attention_layer(layer) else 4
        base = 16 + 16 * layer
        out += [
            Tensor(f"L{layer}.qkv", mb, H + 2 * KVW, H, base + 7),
            Tensor(f"L{layer}.o", mb, H, H, base + 3),
            Tensor(f"L{layer}.gate_up", 4, 2 * F, H, base + 8),
            Tensor(f"L{layer}.down", 4, H, F, base + 6),
        ]
    out.append(Tensor("head", 8, shape.vocab, H, 1023))
    return out


def chain_input_stream(j: int) -> int:
    """j = 0: the embedding row(s); 1 + layer: that layer's mixer output."""
    from . import synth

    return synth.act_stream(CHAIN_INPUT_BASE + j)


def chain_gammas(shape: ChainShape, seed: int):
    """bf16 bits [2 * layers + 1][hidden]: the norm weights, 1 + z / 16."""
    import numpy as np

    from . import synth

    n = 2 * shape.layers + 1
    z = synth.normals_f64(seed, chain_input_stream(1 << 20), 0, n * shape.hidden)
    return synth.f64_to_bf16_bits(1.0 + z / 16.0).reshape(n, shape.hidden)


class DeviceChain:
    """The dependent chain on the current CUDA device: the weights (as in
    DeviceStream), the residual stream h (fp32), the embedding and mixer
    inputs (seeded), the norm weights, every intermediate activation and
    output, and the captured chain (layer_chain_create)."""

    def __init__(self, shape: ChainShape, M: int, seed: int = 0, flags: int = 0):
        import torch

        import bit_weight_gemv_q4_b200 as q4

        from . import synth

        self.shape, self.M, self.seed = shape, M, seed
        H, F, L = shape.hidden, shape.ffn, shape.layers
        self.w = DeviceStream(chain_tensors(shape), M, seed=seed, flags=q4.Q4_STACK_GRAPH)
        self.w.stack.close()
        dev = torch.device("cuda")

        def bf16(n):
            return torch.empty(M * n, dtype=torch.int16, device=dev)

        emb = bf16(H)
        synth.activations_device(seed, chain_input_stream(0), M, H, emb)
        self.emb = emb.view(torch.bfloat16).float()  # the residual stream starts from it (fp32)
        self.h = torch.empty(M * H, dtype=torch.float32, device=dev)
        self.gamma = torch.from_numpy(chain_gammas(shape, seed).view("int16")).to(dev)
        self.x_mix = []
        for layer in range(L):
            xm = bf16(H)
            synth.activations_device(seed, chain_input_stream(1 + layer), M, H, xm)
            self.x_mix.append(xm)
        self.x_qkv = [bf16(H) for _ in range(L)]
        self.x_gu = [bf16(H) for _ in range(L)]
        self.x_down = [bf16(F) for _ in range(L)]
        self.x_head = bf16(H)
        self.ops = self.make_ops()
        torch.cuda.synchronize()
        self.stack = q4.layer_chain_create(self.ops, M, flags)

    def product_index(self, layer: int, which: str) -> int:
        return 4 * layer + {"qkv": 0, "o": 1, "gate_up": 2, "down": 3}[which]

    def make_ops(self):
        import bit_weight_gemv_q4_b200 as q4

        H, F, L = self.shape.hidden, self.shape.ffn, self.shape.layers
        w = self.w
        ops = []

        def product(i, x):
            t = w.tensors[i]
            ops.append((q4.Q4_OP_PRODUCT, t.bits, t.N, t.K, w.packed[i], x, w.y[i], None))

        def norm(y, g, x, first=False):
            ops.append((q4.Q4_OP_RESIDUAL_RMSNORM, 1 if first else 0, H, 0, self.gamma[g], y, x, self.h))

        for layer in range(L):
            prev = self.emb if layer == 0 else w.y[self.product_index(layer - 1, "down")]
            norm(prev, 2 * layer, self.x_qkv[layer], first=layer == 0)
            product(self.product_index(layer, "qkv"), self.x_qkv[layer])
            product(self.product_index(layer, "o"), self.x_mix[layer])
            norm(w.y[self.product_index(layer, "o")], 2 * layer + 1, self.x_gu[layer])
            product(self.product_index(layer, "gate_up"), self.x_gu[layer])
            ops.append((q4.Q4_OP_SWIGLU, 0, F, 0, None, w.y[self.product_index(layer, "gate_up")],
                        self.x_down[layer], None))
            product(self.product_index(layer, "down"), self.x_down[layer])
        last = self.emb if L == 0 else w.y[self.product_index(L - 1, "down")]
        norm(last, 2 * L, self.x_head, first=L == 0)
        product(4 * L, self.x_head)
        return ops

    @property
    def weight_bytes(self) -> int:
        return total_bytes(self.w.tensors)

    @property
    def logits(self):
        return self.w.y[-1]

    def run(self, stream=None) -> None:
        import bit_weight_gemv_q4_b200 as q4

        q4.layer_stack_run(self.stack, stream)

    def check(self, stream=None) -> None:
        import bit_weight_gemv_q4_b200 as q4

        q4.layer_stack_check(self.stack, stream)

    def close(self) -> None:
        self.stack.close()
        self.w.close()
