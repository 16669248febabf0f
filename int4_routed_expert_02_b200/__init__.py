"""int4 routed-expert MoE layer for B200 (sm_100a).

The compute path lives in the C-ABI library `libmoe.so` built from `csrc/`;
`moe` is its thin ctypes binding (argument marshalling only).  `synth`
draws the seeded synthetic inputs.  Importing the package loads nothing;
`int4_routed_expert_02_b200.moe` loads the library and fails loudly when it
is missing.
"""
