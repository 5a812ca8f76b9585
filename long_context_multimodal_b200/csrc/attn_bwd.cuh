// attn_bwd.cuh -- placeholder; the backward kernels are added next.
#pragma once
