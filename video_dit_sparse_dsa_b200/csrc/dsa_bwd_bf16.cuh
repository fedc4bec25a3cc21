// bf16 backward of 3D Deformable Slide Attention (kernels follow).
#pragma once
