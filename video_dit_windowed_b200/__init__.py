"""B200-native (sm_100a) hot path of AtlasVid's detail-branch attention.

``video_dit_windowed_b200.atlas`` binds the C-ABI library ``libatlas.so``
(cube reorder / unorder, 3D RoPE, asymmetric local-global attention).
``video_dit_windowed_b200.workloads`` holds the workload shapes and the seeded
input generator. Importing this package loads nothing; the binding loads the
library on first use and raises if it has not been built.
"""
