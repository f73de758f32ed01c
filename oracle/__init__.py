"""Plain CPU oracle of AutoRound's per-layer SignSGD tuning loop.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package; the library never does, and it shares
no code with the CUDA path (the seeded input generators in ``workloads`` are
the one thing both consume).

Sources, cited by page title and section:

* "[llm-compressor] AutoRound: 부호 경사 하강법으로 라운딩 최적화"
  - section "논문 핵심 내용": RTN  w^ = s*round(w/s);  offset rounding
    w^ = s*round(w/s + V) with V in [-0.5, 0.5];  loss |W^x - Wx|^2;  SignSGD
    V <- V - lr*sign(dL/dV);
  - section "핵심 구조/코드 분석", "on_event with SEQUENTIAL_EPOCH_END": the
    per-layer loop (W taken as fp32, scale/zero-point init by min-max, V = 0,
    forward, MSE, backward, sign update and clamp of V, final fake-quant), and
    ``_fake_quantize_with_offset``  q = clamp(round(W/s + zp + V)), W' = s*(q - zp);
  - section "AutoRoundModifier 생성자 파라미터": iters 200, lr 0.005,
    minmax_lr None -> lr, minmax_shrink 1.0.
* "Introducing AutoRound: Intel's Advanced Quantization for LLMs and VLMs",
  section "2. 반올림과 클리핑 범위의 공동 최적화": rounding and the clipping range
  are tuned jointly by signed gradient descent;  section 4: iters = 0 is RTN.
* "[SGLang] AutoRound: 자동 라운딩 최적화 양자화", section "1. AutoRoundConfig":
  bits in {2, 3, 4, 8}, pack_factor = 32 / bits.

Precision: every quantiser operation (scale, zero-point, the offset rounding,
W', the V/alpha/beta updates) is one IEEE fp32 operation, exactly as the
page's code computes it on ``W.float()``; numpy evaluates each float32
operation with correct rounding and never fuses two.  The layer output, the
loss, the gradient dL/dW' and the straight-through derivatives are computed in
fp64 (the activations are bf16 values, exact in fp64).

Readings where the pages are silent (each also listed in the design notes):
zero-inclusive group min/max; s = 1 for an all-zero group; zp = clamp(rint(.));
symmetric mode s = 2*alpha*amax/Q with zp = 2^(b-1); alpha, beta clamped to
[0.5, 1]; straight-through identity through every rint (zp's included), masked
by clamps with inclusive bounds; sign(0) = 0; one calibration block per step
chosen by a SplitMix64-driven Fisher-Yates permutation per epoch; the state
with the lowest step loss is applied at the end, chosen per output row
(keep_best, the default) or once for the whole layer (keep_best=2); the page's
listing applies the last state, available as keep_best=False; group_size -1 is
one group per row.
"""
from .autoround import (  # noqa: F401
    TuneResult,
    fake_quant,
    layer_mse,
    group_minmax,
    qmax,
    rtn,
    scale_zero_point,
    sign_step,
    step_gradients,
    tune_layer,
)
from .pack import pack_codes, unpack_codes  # noqa: F401
from .schedule import block_schedule, splitmix64_stream  # noqa: F401
from . import chain  # noqa: F401
