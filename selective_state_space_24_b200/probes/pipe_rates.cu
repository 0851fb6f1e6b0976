// pipe_rates.cu -- measures the per-SM issue rates of the pipes the S6 scan
// leans on: MUFU ex2.approx, scalar FFMA, packed FFMA2, and ex2 + FFMA mixed.
// Standalone; not part of libssm.so.
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -o pipe_rates pipe_rates.cu && ./pipe_rates
#include <cstdio>
#include <cuda_runtime.h>
#define ITERS 4096
__device__ __forceinline__ float ex2a(float v){float r;asm volatile("ex2.approx.ftz.f32 %0,%1;":"=f"(r):"f"(v));return r;}
__global__ void k_ex2(float* out, float s){ float x[8]; for(int i=0;i<8;i++) x[i]=threadIdx.x*1e-3f+i*1e-2f;
  for(int it=0;it<ITERS;it++){
#pragma unroll
   for(int i=0;i<8;i++) x[i]=ex2a(x[i]*s);} float r=0; for(int i=0;i<8;i++) r+=x[i]; if(r==123.f) out[0]=r;}
__global__ void k_ffma(float* out, float s){ float x[8]; for(int i=0;i<8;i++) x[i]=threadIdx.x*1e-3f+i;
  for(int it=0;it<ITERS;it++){
#pragma unroll
   for(int i=0;i<8;i++) x[i]=fmaf(x[i],s,0.5f);} float r=0; for(int i=0;i<8;i++) r+=x[i]; if(r==123.f) out[0]=r;}
__global__ void k_ffma2(float* out, float s){ float2 x[8]; for(int i=0;i<8;i++) x[i]=make_float2(threadIdx.x*1e-3f+i, i*0.5f);
  float2 ss=make_float2(s,s), cc=make_float2(0.5f,0.25f);
  for(int it=0;it<ITERS;it++){
#pragma unroll
   for(int i=0;i<8;i++) x[i]=__ffma2_rn(x[i],ss,cc);} float r=0; for(int i=0;i<8;i++) r+=x[i].x+x[i].y; if(r==123.f) out[0]=r;}
// mixed: 8 ex2 chains + 16 ffma chains per iteration
__global__ void k_mix(float* out, float s){ float x[8], y[16]; for(int i=0;i<8;i++) x[i]=threadIdx.x*1e-3f+i*1e-2f; for(int i=0;i<16;i++) y[i]=i;
  for(int it=0;it<ITERS;it++){
#pragma unroll
   for(int i=0;i<8;i++) x[i]=ex2a(x[i]*s);
#pragma unroll
   for(int i=0;i<16;i++) y[i]=fmaf(y[i],s,0.5f);}
  float r=0; for(int i=0;i<8;i++) r+=x[i]; for(int i=0;i<16;i++) r+=y[i]; if(r==123.f) out[0]=r;}
int main(){
  float* d; cudaMalloc(&d, 16);
  int dev; cudaGetDevice(&dev); int clk; cudaDeviceGetAttribute(&clk, cudaDevAttrClockRate, dev);
  int sms; cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  dim3 g(sms*8), b(256);
  cudaEvent_t e0,e1; cudaEventCreate(&e0); cudaEventCreate(&e1);
  const char* names[]={"ex2.approx.f32 (+FMUL)","FFMA","FFMA2 (2 ops/lane)","8 ex2(+FMUL) + 16 FFMA"};
  double ops_per_iter_thread[]={8,8,16,8};
  for(int k=0;k<4;k++){
    for(int rep=0;rep<2;rep++){
      cudaEventRecord(e0);
      if(k==0) k_ex2<<<g,b>>>(d,0.999f); else if(k==1) k_ffma<<<g,b>>>(d,0.999f); else if(k==2) k_ffma2<<<g,b>>>(d,0.999f); else k_mix<<<g,b>>>(d,0.999f);
      cudaEventRecord(e1); cudaEventSynchronize(e1);
      float ms; cudaEventElapsedTime(&ms,e0,e1);
      double ops=(double)g.x*b.x*ITERS*ops_per_iter_thread[k];
      if(rep==1) printf("%-28s %8.3f ms  %8.1f Gop/s  %6.2f per clk per SM at %d MHz (primary op)\n", names[k], ms, ops/ms/1e6, ops/(ms*1e-3)/(clk*1e3)/sms, clk/1000);
    }
  }
  cudaError_t e=cudaGetLastError(); printf("err=%s\n", cudaGetErrorString(e)); return e!=cudaSuccess;
}
