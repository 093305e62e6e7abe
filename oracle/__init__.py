"""The oracle: a plain fp64 C restatement of the quantized MoE FFN step.
Test infrastructure only; the library's code path never imports it."""
