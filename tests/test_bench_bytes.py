"""The algorithmic byte counts behind the bench's GB/s figures, against totals worked by hand
from the data layout (Mamba-2 1.3B: d_model 2048, d_inner 4096, 64 heads of 64 channels,
d_state 128, 4 taps, 48 blocks, a 50,288-row int8 table).

State step, one layer, one token:
  in_proj output in   8,512 bf16                         =    17,024
  shift register      4,352 channels x 4 taps bf16, in + out =    69,632
  SSM state           64 x 64 x 128 fp32, in + out         = 4,194,304
  out                 4,096 bf16                           =     8,192
  parameters          fp32: conv w 17,408 + conv b 4,352 + dt_bias, a_log, D 3 x 64
                      + norm w 4,096 = 26,048 values        =   104,192
  per layer 4,393,344; 48 layers 210,880,512.
Chained decode step, one token:
  the 96 linears (stack)                                     173,420,544
  48 state steps                                             210,880,512
  49 residual add + RMS norms: w 8,192 + r in 8,192 + delta 4,096 + r out 8,192 + out 4,096
                                = 32,768 each                  1,605,632
  LM head: table 102,989,824 + scales 201,152 + h 4,096 + fp32 logits 201,152 = 103,396,224
  embedding: row 2,048 + scale 4 + fp32 out 8,192 + id 4          10,248
  total                                                      489,313,160
"""
import bench
import dfssm_synth as synth


def test_state_step_bytes():
    assert bench.ssm_layer_bytes(synth.SSM_DIMS, 1) == 4_393_344
    assert 48 * bench.ssm_layer_bytes(synth.SSM_DIMS, 1) == 210_880_512


def test_chained_decode_step_bytes():
    assert bench.chain_bytes(48, synth.D_MODEL, synth.SSM_DIMS, synth.VOCAB, 1) == 489_313_160
