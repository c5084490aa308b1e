"""Torch-facing calls of the ternary BitLinear path.

Each function checks dtype, device and contiguity, allocates its outputs with
torch (device memory is torch's job here), and hands raw pointers to one C
entry point of libbitlinear.so.  All arithmetic runs in the CUDA kernels;
nothing here falls back to the CPU.
"""
import torch

from . import _lib

# Largest token count the CUDA-core GEMV handles.
GEMV_MAX_TOKENS = 16

# Smallest token count for which `matmul` and `TernaryLinear` use the
# tensor-core GEMM.  Measured on B200 on an 8B-shaped layer (7 projections,
# one grouped launch, weights not in L2): GEMV 24.6 / 30.1 / 40.8 / 54.9 /
# 104 us and GEMM 24.5 / 24.6 / 24.6 / 24.3 / 24.3 us at N = 1 / 2 / 4 / 8 /
# 16; from fp32 activations, the fused quantise+GEMV 26.8 / 38.4 us at N = 1 /
# 2.  The two tie at one token; from two on, the GEMV's per-token dp4a work
# costs more than the GEMM's whole launch.
GEMM_MIN_TOKENS = 2


def _need(t, dtype, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (no CPU path exists)" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _on(device, **tensors):
    """Every given tensor (None skipped) must sit on `device`: the kernels run
    on one GPU and dereference all pointers there."""
    for name, t in tensors.items():
        if t is not None and t.device != device:
            raise ValueError("%s is on %s, the weights on %s: all operands must share one "
                             "device" % (name, t.device, device))


def _check_out(out, N, M, device, name="out"):
    """A caller-supplied output must be fp32 [N, M], contiguous, on `device`
    (the kernels write N*M floats through its pointer)."""
    if out is None:
        return
    if not isinstance(out, torch.Tensor) or tuple(out.shape) != (N, M):
        raise ValueError("%s must have shape (%d, %d), got %s"
                         % (name, N, M, tuple(getattr(out, "shape", ()))))
    _need(out, torch.float32, name)
    _on(device, **{name: out})


def _check_token_vector(t, N, dtype, name):
    """amax / xsum: one entry per token, read for every n < N."""
    _need(t, dtype, name)
    if t.numel() != N:
        raise ValueError("%s must hold N = %d entries, got %d" % (name, N, t.numel()))


def packed_row_words(K):
    """Words per packed row: K/16 rounded up to a multiple of 4 (rows end on a
    16-byte boundary; the padding fields hold code 0)."""
    return 4 * ((K + 63) // 64)


def pack_weights(W, stream=None):
    """fp32 W[M,K] -> (packed int32 [M, packed_row_words(K)] holding the uint32
    words, alpha fp32 [1])."""
    _need(W, torch.float32, "W")
    M, K = W.shape
    packed = torch.empty((M, packed_row_words(K)), dtype=torch.int32, device=W.device)
    alpha = torch.empty(1, dtype=torch.float32, device=W.device)
    nbytes = _lib.bitlinear_pack_workspace_bytes(M, K)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    _lib.check(_lib.bitlinear_pack_weights(W, M, K, packed, alpha, ws, nbytes, stream),
               "bitlinear_pack_weights")
    return packed, alpha


def quant_act(x, stream=None, with_sum=True):
    """fp32 x[N,K] -> (xq int8 [N,K], amax fp32 [N], xsum int32 [N] or None)."""
    _need(x, torch.float32, "x")
    N, K = x.shape
    xq = torch.empty((N, K), dtype=torch.int8, device=x.device)
    amax = torch.empty(N, dtype=torch.float32, device=x.device)
    xsum = torch.empty(N, dtype=torch.int32, device=x.device) if with_sum else None
    _lib.check(_lib.bitlinear_quant_act(x, N, K, xq, amax, xsum, stream), "bitlinear_quant_act")
    return xq, amax, xsum


def quant_act_per_tensor(x, stream=None):
    """Per-tensor variant: one absmax over all of x; amax[n] holds it for every n."""
    _need(x, torch.float32, "x")
    N, K = x.shape
    xq = torch.empty((N, K), dtype=torch.int8, device=x.device)
    amax = torch.empty(N, dtype=torch.float32, device=x.device)
    xsum = torch.empty(N, dtype=torch.int32, device=x.device)
    nbytes = _lib.load().bitlinear_quant_act_per_tensor_workspace_bytes()
    ws = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    _lib.check(_lib.bitlinear_quant_act_per_tensor(x, N, K, xq, amax, xsum, ws, nbytes, stream),
               "bitlinear_quant_act_per_tensor")
    return xq, amax, xsum


def quant_act_grouped(xs, stream=None):
    """Quantise several fp32 activation matrices in one launch; returns a list
    of (xq, amax, xsum)."""
    outs, entries = [], []
    for x in xs:
        _need(x, torch.float32, "x")
        N, K = x.shape
        o = (torch.empty((N, K), dtype=torch.int8, device=x.device),
             torch.empty(N, dtype=torch.float32, device=x.device),
             torch.empty(N, dtype=torch.int32, device=x.device))
        outs.append(o)
        entries.append((x,) + o)
    arr = _lib.make_acts(entries)
    _lib.check(_lib.bitlinear_quant_act_grouped(arr, len(entries), stream),
               "bitlinear_quant_act_grouped")
    return outs


def _matmul(fn, name, packed, alpha, xq, amax, xsum, M, with_acc, stream, out=None):
    _need(packed, torch.int32, "packed")
    _need(alpha, torch.float32, "alpha")
    _need(xq, torch.int8, "xq")
    N, K = xq.shape
    _check_token_vector(amax, N, torch.float32, "amax")
    _check_token_vector(xsum, N, torch.int32, "xsum")
    if packed.shape != (M, packed_row_words(K)):
        raise ValueError("packed must be [M, packed_row_words(K)] = [%d, %d], got %s"
                         % (M, packed_row_words(K), tuple(packed.shape)))
    dev = packed.device
    _on(dev, alpha=alpha, xq=xq, amax=amax, xsum=xsum)
    _check_out(out, N, M, dev)
    y = out if out is not None else torch.empty((N, M), dtype=torch.float32, device=dev)
    acc = torch.empty((N, M), dtype=torch.int32, device=dev) if with_acc else None
    with torch.cuda.device(dev):
        _lib.check(fn(packed, alpha, M, K, xq, amax, xsum, N, y, acc, stream), name)
    return (y, acc) if with_acc else y


def gemv(packed, alpha, xq, amax, xsum, M=None, with_acc=False, stream=None, out=None):
    """Decode GEMV (N <= 16): y[N,M] fp32 (and int32 acc if with_acc)."""
    M = packed.shape[0] if M is None else M
    return _matmul(_lib.bitlinear_gemv, "bitlinear_gemv", packed, alpha, xq, amax, xsum, M,
                   with_acc, stream, out)


def _grouped(fn, name, layers, xq, amax, xsum, with_acc, stream, outs):
    n = len(layers)
    xqs = xq if isinstance(xq, (list, tuple)) else [xq] * n
    amaxs = amax if isinstance(amax, (list, tuple)) else [amax] * n
    xsums = xsum if isinstance(xsum, (list, tuple)) else [xsum] * n
    if not (len(xqs) == len(amaxs) == len(xsums) == n) or (outs is not None and len(outs) != n):
        raise ValueError("one xq, amax, xsum (and out) per layer, or one for all")
    N = xqs[0].shape[0]
    dev = layers[0][0].device if n else None
    ys, accs, entries = [], [], []
    for i, (packed, alpha) in enumerate(layers):
        _need(packed, torch.int32, "packed")
        _need(alpha, torch.float32, "alpha")
        _need(xqs[i], torch.int8, "xq")
        _check_token_vector(amaxs[i], N, torch.float32, "amax")
        _check_token_vector(xsums[i], N, torch.int32, "xsum")
        M, K = packed.shape[0], xqs[i].shape[1]
        if xqs[i].shape[0] != N or packed.shape[1] != packed_row_words(K):
            raise ValueError("layer %d: packed [M, packed_row_words(K)] must match xq [N, K];"
                             " N shared" % i)
        _on(dev, packed=packed, alpha=alpha, xq=xqs[i], amax=amaxs[i], xsum=xsums[i])
        if outs is not None:
            _check_out(outs[i], N, M, dev, "outs[%d]" % i)
        y = outs[i] if outs is not None else torch.empty((N, M), dtype=torch.float32,
                                                           device=dev)
        acc = torch.empty((N, M), dtype=torch.int32, device=dev) if with_acc else None
        ys.append(y)
        accs.append(acc)
        entries.append((packed, alpha, M, K, xqs[i], amaxs[i], xsums[i], y, acc))
    arr = _lib.make_problems(entries)
    if n:
        with torch.cuda.device(dev):
            _lib.check(fn(arr, n, N, stream), name)
    return (ys, accs) if with_acc else ys


def gemv_grouped(layers, xq, amax, xsum, with_acc=False, stream=None, outs=None):
    """One grouped decode call over several layers sharing the token count.
    layers: list of (packed, alpha); xq/amax/xsum: one tensor for all layers or
    a list with one entry per layer (K may differ between layers).  Returns a
    list of y (and of acc)."""
    return _grouped(_lib.bitlinear_gemv_grouped, "bitlinear_gemv_grouped", layers, xq, amax,
                    xsum, with_acc, stream, outs)


def gemm_grouped(layers, xq, amax, xsum, with_acc=False, stream=None, outs=None):
    """Tensor-core GEMM over several layers in one persistent launch; same
    arguments as gemv_grouped."""
    return _grouped(_lib.bitlinear_gemm_grouped, "bitlinear_gemm_grouped", layers, xq, amax,
                    xsum, with_acc, stream, outs)


def gemm(packed, alpha, xq, amax, xsum, M=None, with_acc=False, stream=None, out=None):
    """Tensor-core GEMM (any N and M): y[N,M] fp32 (and int32 acc)."""
    M = packed.shape[0] if M is None else M
    return _matmul(_lib.bitlinear_gemm, "bitlinear_gemm", packed, alpha, xq, amax, xsum, M,
                   with_acc, stream, out)


def matmul(packed, alpha, xq, amax, xsum, M=None, with_acc=False, stream=None, out=None):
    """GEMV below GEMM_MIN_TOKENS tokens, else the tensor-core GEMM."""
    M = packed.shape[0] if M is None else M
    if xq.shape[0] < GEMM_MIN_TOKENS:
        return gemv(packed, alpha, xq, amax, xsum, M, with_acc, stream, out)
    return gemm(packed, alpha, xq, amax, xsum, M, with_acc, stream, out)


# Shared-memory bound of the fused decode kernel: tokens x K rounded up to 512.
GEMV_QUANT_MAX_BYTES = 65536


def gemv_quant_fits(N, K):
    """Whether the fused quantise+GEMV kernel takes N tokens of width K."""
    return 1 <= N <= GEMV_MAX_TOKENS and N * (-(-K // 512) * 512) <= GEMV_QUANT_MAX_BYTES


def use_fused_decode(N, K):
    """TernaryLinear's choice: the fused kernel below the GEMM crossover."""
    return N < GEMM_MIN_TOKENS and gemv_quant_fits(N, K)


def gemv_quant(packed, alpha, x, M=None, with_acc=False, stream=None, out=None):
    """Decode GEMV straight from fp32 activations x[N,K] (N <= 16): the kernel
    quantises x per token itself.  Same y (and acc) as quant_act + gemv."""
    _need(packed, torch.int32, "packed")
    _need(alpha, torch.float32, "alpha")
    _need(x, torch.float32, "x")
    M = packed.shape[0] if M is None else M
    N, K = x.shape
    if packed.shape != (M, packed_row_words(K)):
        raise ValueError("packed must be [M, packed_row_words(K)] = [%d, %d], got %s"
                         % (M, packed_row_words(K), tuple(packed.shape)))
    dev = packed.device
    _on(dev, alpha=alpha, x=x)
    _check_out(out, N, M, dev)
    y = out if out is not None else torch.empty((N, M), dtype=torch.float32, device=dev)
    acc = torch.empty((N, M), dtype=torch.int32, device=dev) if with_acc else None
    with torch.cuda.device(dev):
        _lib.check(_lib.bitlinear_gemv_quant(packed, alpha, M, K, x, N, y, acc, stream),
                   "bitlinear_gemv_quant")
    return (y, acc) if with_acc else y


def gemv_quant_grouped(layers, x, with_acc=False, stream=None, outs=None):
    """Fused decode over several layers in one launch.  layers: list of
    (packed, alpha); x: one fp32 tensor [N,K] for all layers or a list with
    one per layer.  Layers that share an input should pass the same tensor and
    be adjacent, so that the kernel quantises it once for the rows it streams.
    Returns a list of y (and of acc)."""
    n = len(layers)
    xs = x if isinstance(x, (list, tuple)) else [x] * n
    if len(xs) != n or (outs is not None and len(outs) != n):
        raise ValueError("one x (and out) per layer, or one x for all")
    N = xs[0].shape[0]
    dev = layers[0][0].device if n else None
    ys, accs, entries = [], [], []
    for i, (packed, alpha) in enumerate(layers):
        _need(packed, torch.int32, "packed")
        _need(alpha, torch.float32, "alpha")
        _need(xs[i], torch.float32, "x")
        M, K = packed.shape[0], xs[i].shape[1]
        if xs[i].shape[0] != N or packed.shape[1] != packed_row_words(K):
            raise ValueError("layer %d: packed [M, packed_row_words(K)] must match x [N, K];"
                             " N shared" % i)
        _on(dev, packed=packed, alpha=alpha, x=xs[i])
        if outs is not None:
            _check_out(outs[i], N, M, dev, "outs[%d]" % i)
        y = outs[i] if outs is not None else torch.empty((N, M), dtype=torch.float32,
                                                           device=dev)
        acc = torch.empty((N, M), dtype=torch.int32, device=dev) if with_acc else None
        ys.append(y)
        accs.append(acc)
        entries.append((packed, alpha, M, K, xs[i], y, acc))
    arr = _lib.make_fused_problems(entries)
    if n:
        with torch.cuda.device(dev):
            _lib.check(_lib.bitlinear_gemv_quant_grouped(arr, n, N, stream),
                       "bitlinear_gemv_quant_grouped")
    return (ys, accs) if with_acc else ys


def tl2_row_bytes(K):
    """Bytes of one TL2-style row (5 bits per three weights, see include/bitlinear.h)."""
    n = _lib.load().bitlinear_tl2_row_bytes(int(K))
    if n == 0:
        raise ValueError("K must be a positive multiple of 16, at most 131072")
    return n


def tl2_from_packed(packed, K, stream=None):
    """Re-encode 2-bit packed weights [M, packed_row_words(K)] as TL2-style
    rows: uint8 [M, tl2_row_bytes(K)]."""
    _need(packed, torch.int32, "packed")
    M = packed.shape[0]
    if packed.shape[1] != packed_row_words(K):
        raise ValueError("packed must be [M, packed_row_words(K)]")
    out = torch.empty((M, tl2_row_bytes(K)), dtype=torch.uint8, device=packed.device)
    _lib.check(_lib.bitlinear_tl2_from_packed(packed, M, K, out, stream),
               "bitlinear_tl2_from_packed")
    return out


def gemv_tl2(tl2, alpha, xq, amax, M=None, with_acc=False, stream=None, out=None):
    """Decode GEMV over TL2-style rows (N <= 16): same y (and acc) as gemv."""
    _need(tl2, torch.uint8, "tl2")
    _need(alpha, torch.float32, "alpha")
    _need(xq, torch.int8, "xq")
    M = tl2.shape[0] if M is None else M
    N, K = xq.shape
    _check_token_vector(amax, N, torch.float32, "amax")
    if tl2.shape != (M, tl2_row_bytes(K)):
        raise ValueError("tl2 must be [M, tl2_row_bytes(K)] = [%d, %d]" % (M, tl2_row_bytes(K)))
    dev = tl2.device
    _on(dev, alpha=alpha, xq=xq, amax=amax)
    _check_out(out, N, M, dev)
    y = out if out is not None else torch.empty((N, M), dtype=torch.float32, device=dev)
    acc = torch.empty((N, M), dtype=torch.int32, device=dev) if with_acc else None
    with torch.cuda.device(dev):
        _lib.check(_lib.bitlinear_gemv_tl2(tl2, alpha, M, K, xq, amax, N, y, acc, stream),
                   "bitlinear_gemv_tl2")
    return (y, acc) if with_acc else y


class TernaryLinear:
    """A BitLinear layer: packed 2-bit ternary weights + alpha, applied to fp32
    activations: the fused quantise+GEMV kernel below GEMM_MIN_TOKENS tokens,
    else quant_act -> tensor-core GEMM with the fused rescale."""

    def __init__(self, packed, alpha, in_features, out_features):
        self.packed, self.alpha = packed, alpha
        self.in_features, self.out_features = in_features, out_features

    @classmethod
    def from_float(cls, W, stream=None):
        packed, alpha = pack_weights(W, stream)
        return cls(packed, alpha, W.shape[1], W.shape[0])

    def __call__(self, x, stream=None):
        if use_fused_decode(x.shape[0], x.shape[1]):
            return gemv_quant(self.packed, self.alpha, x, self.out_features, stream=stream)
        xq, amax, xsum = quant_act(x, stream)
        return matmul(self.packed, self.alpha, xq, amax, xsum, self.out_features, stream=stream)
