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
values, N*K/16: the same 4.5 bits per weight as q4.  q5 and q6 tensors hold
N*K*5/8 or N*K*6/8 code bytes plus the fp16 scales.
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
    codes = N * K * bits // 8  # q4, q5, q6, q8
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


def as_width(tensors: list[Tensor], bits: int) -> list[Tensor]:
    """The same list with every q4 tensor at another width (5 or 6 bits; the
    q8 tensors kept)."""
    return [Tensor(t.name, bits, t.N, t.K, t.tensor_id) if t.bits == 4 else t for t in tensors]


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
        max_canon = max((t.N * (t.K // 2 if t.bits in (4, NVFP4) else t.K) for t in self.tensors), default=0)
        max_scales = max((t.N * (t.K // 16 if t.bits == NVFP4 else t.K // 32 * 2) for t in self.tensors), default=0)
        canon = torch.empty(max(max_canon, 16), dtype=torch.uint8, device=dev)
        scales = torch.empty(max(max_scales, 16), dtype=torch.uint8, device=dev)
        self.packed = []
        for t in self.tensors:
            nq = t.N * (t.K // 2 if t.bits in (4, NVFP4) else t.K)
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


# ----------------------------------------------------------------------------
# One speculative decoding step around the M = 4 pass (bs178.com llamAmpere
# post, "Why it is this fast", part four): three draft tokens, each from the
# draft head's projection onto a vocabulary map of 65,536 tokens followed by a
# draw, then one pass of the main model's stream at M = 4 (the three drafts
# plus one), whose output head gives the target logits, then the keep /
# reject step.  The MTP layer that turns a drafted token into the next draft
# hidden state needs trained weights and is not computed: each draft's hidden
# state is a seeded input.
# ----------------------------------------------------------------------------
SPEC_DRAFTS = 3
SPEC_INPUT_BASE = 1 << 25  # generator streams of the step's own inputs


def vocab_map(seed: int, V: int = VOCAB, n_map: int = DRAFT_VOCAB):
    """A synthetic vocabulary map (the pages' map file is not available):
    n_map distinct token ids, ascending, chosen by seeded random keys."""
    import numpy as np

    from . import synth

    keys = synth.words(seed, synth.act_stream(SPEC_INPUT_BASE), 0, V)
    return np.sort(np.argsort(keys, kind="stable")[:n_map]).astype(np.int32)


def spec_uniforms(seed: int, count: int):
    """Seeded uniforms in [0, 1) (fp32) for the draws of a step."""
    import numpy as np

    from . import synth

    w = synth.words(seed, synth.act_stream(SPEC_INPUT_BASE + 1), 0, count)
    return ((w >> np.uint64(40)).astype(np.float64) / float(1 << 24)).astype(np.float32)


class DeviceSpec:
    """The speculative step on the current CUDA device: the verify stream
    (DeviceStream of the decode stream at M = n + 1), the mapped draft head
    (the head's rows at the map's tokens, gathered and packed on the device),
    one single-product stack per draft, the draft hidden states, logits,
    drawn rows, uniforms and the verify output."""

    def __init__(self, seed: int = 0, temperature: float = 1.0, n_draft: int = SPEC_DRAFTS):
        import torch

        import bit_weight_gemv_q4_b200 as q4

        from . import synth

        self.seed, self.T, self.n = seed, float(temperature), n_draft
        dev = torch.device("cuda")
        tensors = decode_stream(fused=True)
        head = tensors[-1]
        self.V, self.K = head.N, head.K
        self.verify_stream = DeviceStream(tensors, n_draft + 1, seed=seed, flags=q4.Q4_STACK_INDEPENDENT)
        self.vmap_host = vocab_map(seed, self.V)
        self.n_map = len(self.vmap_host)
        self.vmap = torch.from_numpy(self.vmap_host).to(dev)
        inv = torch.full((self.V,), -1, dtype=torch.int32)
        inv[torch.from_numpy(self.vmap_host).long()] = torch.arange(self.n_map, dtype=torch.int32)
        self.inv_map = inv.to(dev)
        # the mapped draft head: the head's canonical rows at the map's tokens
        canon = torch.empty(self.V * self.K, dtype=torch.uint8, device=dev)
        scales = torch.empty(self.V * (self.K // 32), dtype=torch.int16, device=dev)
        synth.weights_device(8, seed, synth.weight_stream(head.tensor_id), self.K, 0, self.V, canon)
        synth.scales_device(seed, synth.scale_stream(head.tensor_id), self.K, 0, self.V, scales)
        gq = torch.empty(self.n_map * self.K, dtype=torch.uint8, device=dev)
        gs = torch.empty(self.n_map * (self.K // 32), dtype=torch.int16, device=dev)
        q4.q4_gather_rows_device(canon, self.K, self.V, self.vmap, self.n_map, gq)
        q4.q4_gather_rows_device(scales, 2 * (self.K // 32), self.V, self.vmap, self.n_map, gs)
        self.draft_packed = torch.empty(q4.q4_packed_bytes(8, self.n_map, self.K), dtype=torch.uint8, device=dev)
        q4.q4_pack_weights_device(8, gq, gs, self.n_map, self.K, self.draft_packed)
        del canon, scales, gq, gs
        self.x_draft = []
        for j in range(n_draft):
            xj = torch.empty(self.K, dtype=torch.int16, device=dev)
            synth.activations_device(seed, synth.act_stream(SPEC_INPUT_BASE + 2 + j), 1, self.K, xj)
            self.x_draft.append(xj)
        self.z = torch.empty(max(n_draft, 1) * self.n_map, dtype=torch.float32, device=dev)
        self.draft_stacks = [
            q4.layer_stack_create([(8, self.n_map, self.K, self.draft_packed, self.x_draft[j],
                                    self.z[j * self.n_map:(j + 1) * self.n_map])], 1, q4.Q4_STACK_INDEPENDENT)
            for j in range(n_draft)]
        self.u_host = spec_uniforms(seed, 3 * n_draft + 1)
        self.u = torch.from_numpy(self.u_host).to(dev)
        self.rows = torch.zeros(max(n_draft, 1), dtype=torch.int32, device=dev)
        self.tokens = torch.zeros(max(n_draft, 1), dtype=torch.int32, device=dev)
        self.q = torch.zeros(max(n_draft, 1), dtype=torch.float32, device=dev)
        self.out = torch.zeros(3 * n_draft + 3, dtype=torch.int32, device=dev)
        torch.cuda.synchronize()

    @property
    def target_logits(self):
        return self.verify_stream.y[-1]  # [n + 1][V]

    def draft(self, j: int, stream=None) -> None:
        import bit_weight_gemv_q4_b200 as q4

        q4.layer_stack_run(self.draft_stacks[j], stream)
        q4.q4_spec_draft(self.z[j * self.n_map:(j + 1) * self.n_map], self.n_map, self.vmap, self.T,
                         self.u[j:j + 1], self.rows[j:j + 1], self.tokens[j:j + 1], self.q[j:j + 1], stream)

    def verify(self, stream=None) -> None:
        import bit_weight_gemv_q4_b200 as q4

        q4.q4_spec_verify(self.target_logits, self.V, self.z, self.n_map, self.vmap, self.inv_map, self.rows,
                          self.n, self.T, self.u[self.n:], self.out, stream)

    def run(self, stream=None) -> None:
        """One step: the drafts, the M = n + 1 pass, the keep / reject step."""
        for j in range(self.n):
            self.draft(j, stream)
        self.verify_stream.run(stream)
        self.verify(stream)

    def check(self, stream=None) -> None:
        import bit_weight_gemv_q4_b200 as q4

        for st in self.draft_stacks:
            q4.layer_stack_check(st, stream)
        self.verify_stream.check(stream)

    def close(self) -> None:
        for st in self.draft_stacks:
            st.close()
        self.draft_stacks.clear()
        self.verify_stream.close()
